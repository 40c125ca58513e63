"""Property tests of the host layout (no GPU): for random configurations the
partitions tile the state, the stage-3 units tile the flat vector in order,
the transient buffer is the largest unit, and the ledger equals the oracle's
(with K = 12, or K = 8 without fp32 master weights: [P1] "Where 16 bytes per
parameter comes from", [P3] "Why parameter count is not training memory")."""
import numpy as np
from hypothesis import given, settings
from hypothesis import strategies as st

from oracle import zero_ref as Z
from zero_partitioned_mixed_02_b200 import _abi as A


@st.composite
def configs(draw):
    nd = draw(st.integers(1, 40))
    n_t = draw(st.integers(1, 12))
    numel = draw(st.lists(st.integers(1, 5000), min_size=n_t, max_size=n_t))
    units, u = [], 0
    for i in range(n_t):
        if i > 0 and draw(st.booleans()):
            u += 1
        units.append(u)
    flags = draw(st.lists(st.sampled_from([0, A.ZERO_TENSOR_NO_DECAY]), min_size=n_t, max_size=n_t))
    stage = draw(st.integers(1, 3))
    variant = draw(st.sampled_from([A.ZERO_VARIANT_FUSED, A.ZERO_VARIANT_TWO_PASS, A.ZERO_VARIANT_FUSED_TMA,
                                    A.ZERO_VARIANT_TWO_PASS_TMA]))
    bf16 = draw(st.booleans()) and variant in (A.ZERO_VARIANT_TWO_PASS, A.ZERO_VARIANT_TWO_PASS_TMA)
    return nd, list(zip(numel, units, flags)), stage, variant, bf16


@settings(max_examples=300, deadline=None)
@given(configs())
def test_layout_invariants(c):
    nd, tensors, stage, variant, bf16 = c
    psi = sum(t[0] for t in tensors)
    cfg = A.Config(psi, nd, stage, variant=variant, tensors=tensors,
                   precision=A.ZERO_PRECISION_BF16 if bf16 else A.ZERO_PRECISION_FP16)
    L = A.zero_state_bytes(cfg)
    numel = [t[0] for t in tensors]
    # shards tile the state in rank order
    pos = 0
    for r in range(nd):
        b, n = A.zero_rank_shard(cfg, r)
        assert b == pos
        want = (Z.shard_len(numel, nd, r) if stage == 3 else
                (lambda be: be[1] - be[0])(Z.partition(psi, nd, r)))
        assert n == want
        pos += n
    assert pos == L.state_elems == psi
    # ledger: the oracle's exact bytes with K = 12, or K = 8 without master
    ex = Z.ledger_exact(psi, nd, numel)
    if bf16:
        P = max(e - b for b, e in (Z.partition(psi, nd, r) for r in range(nd)))
        S = max(Z.shard_len(numel, nd, r) for r in range(nd))
        ex = [12 * psi, 4 * psi + 8 * P, 2 * psi + 10 * P, 12 * S]
    assert list(L.exact_bytes) == list(ex)
    assert list(L.comm_elements) == list(Z.comm_elements(psi, nd).values())
    if stage == 3:
        # units tile the flat vector in order; the transient is the largest
        flat, biggest = 0, 0
        for u in range(L.n_units):
            fb, cnt = A.zero_unit_range(cfg, u)
            assert fb == flat
            assert cnt == sum(n for n, uu, _ in tensors if uu == u)
            flat += cnt
            biggest = max(biggest, cnt)
        assert flat == psi
        assert L.transient_bytes == 2 * biggest
        assert L.peak_stage3_bytes == L.exact_bytes[3] + 2 * biggest
    # the workspace holds every region
    assert L.workspace_bytes >= (8 if bf16 else 12) * psi * (1 if variant in (1, 3) else 2)
    if not bf16:
        o = A.zero_offload_bytes(cfg, 256)
        assert o.state_elems == psi and o.host_state_bytes == 12 * psi
        assert o.n_chunks == -(-psi // o.chunk_elems)


@settings(max_examples=200, deadline=None)
@given(configs(), st.integers(0, 39))
def test_stage3_rank_view(c, r):
    """Rank r of a real stage-3 job: its state is shard r (the oracle's shard
    length), gradients stay full length, the ledger is the job's, and the
    workspace holds the shard plus the gather tables; an offloaded stage-3
    rank and a stage-3 rank with Nd outputs are refused."""
    nd, tensors, _, variant, bf16 = c
    r = r % nd
    psi = sum(t[0] for t in tensors)
    prec = A.ZERO_PRECISION_BF16 if bf16 else A.ZERO_PRECISION_FP16
    job = A.zero_state_bytes(A.Config(psi, nd, 3, variant=variant, tensors=tensors, precision=prec))
    cfg = A.Config(psi, nd, 3, rank_view=r, variant=variant, tensors=tensors, precision=prec)
    L = A.zero_state_bytes(cfg)
    assert L.state_elems == Z.shard_len([t[0] for t in tensors], nd, r)
    # the handle holds shard r alone, from 0
    assert [A.zero_rank_shard(cfg, k) for k in range(nd)] == [(0, L.state_elems if k == r else 0)
                                                             for k in range(nd)]
    assert L.grad_len == psi
    assert list(L.exact_bytes) == list(job.exact_bytes) and L.transient_bytes == job.transient_bytes
    assert L.off_shard16 > 0 and L.off_shard16 + 2 * L.state_elems <= L.workspace_bytes
    if nd > 1:
        try:
            A.zero_state_bytes(A.Config(psi, nd, 3, rank_view=r, variant=variant, tensors=tensors,
                                        precision=prec, view_outputs=nd))
            raise AssertionError("a stage-3 rank with Nd outputs was accepted")
        except A.ZeroError as e:
            assert e.code == A.ZERO_ERR_ARG
    try:
        A.zero_offload_bytes(A.Config(psi, nd, 3, rank_view=r, tensors=tensors))
        raise AssertionError("an offloaded stage-3 rank was accepted")
    except A.ZeroError as e:
        assert e.code == A.ZERO_ERR_ARG


@settings(max_examples=200, deadline=None)
@given(configs(), st.integers(-1, 39))
def test_gather_plan_against_the_oracles_chunks(c, view):
    """The stage-3 gather plan (zero_gather_plan: what the rank gather runs)
    copies, for every tensor of a unit and every rank in order, the oracle's
    chunk of that tensor from the rank's shard: the source offset is the
    rank's earlier chunks, the destination the chunk's place in the unit, and
    the runs tile the unit."""
    nd, tensors, _, variant, _ = c
    view = view % nd if view >= 0 else -1
    numel = [t[0] for t in tensors]
    unit_of = [t[1] for t in tensors]
    psi = sum(numel)
    cfg = A.Config(psi, nd, 3, rank_view=view, variant=variant, tensors=tensors)
    def chunk_len(t, r):
        b, e = Z.chunk(numel[t], nd, r)
        return e - b

    def in_shard(t, r):  # rank r's chunks of the tensors before t
        return sum(chunk_len(k, r) for k in range(t))

    for u in range(unit_of[-1] + 1):
        flat0 = A.zero_unit_range(cfg, u)[0]
        want = []
        for t in (k for k in range(len(numel)) if unit_of[k] == u):
            for r in range(nd):
                b, e = Z.chunk(numel[t], nd, r)
                if e > b:
                    want.append((r, in_shard(t, r), sum(numel[:t]) - flat0 + b, e - b))
        plan = A.zero_gather_plan(cfg, u)
        assert plan == want
        # tiling, and every source range inside its rank's shard
        assert sum(x[3] for x in plan) == A.zero_unit_range(cfg, u)[1]
        pos = 0
        for r, sb, ob, n in plan:
            assert ob == pos and n > 0 and 0 <= sb and sb + n <= Z.shard_len(numel, nd, r)
            pos += n
    try:
        A.zero_gather_plan(A.Config(psi, nd, 2, variant=variant, tensors=tensors), 0)
        raise AssertionError("a stage-2 plan was given")
    except A.ZeroError as e:
        assert e.code == A.ZERO_ERR_STAGE
