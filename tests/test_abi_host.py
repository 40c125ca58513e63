"""Host-only checks of the C ABI (no GPU needed): the library loads and
exports every symbol include/*.h declares; the ledger, partition and unit
queries equal the oracle's; argument validation returns the documented codes
before any device work.
"""
import ctypes as C
import glob
import os
import re

import numpy as np
import pytest

from oracle import zero_ref as Z
from zero_partitioned_mixed_02_b200 import _abi as A
from zero_partitioned_mixed_02_b200.synth import workloads as W

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    names = set()
    for path in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = open(path).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        src = re.sub(r"//[^\n]*", "", src)
        for m in re.finditer(r"^\s*(?:const\s+)?[A-Za-z_][\w\s\*]*?\b(zero_\w+)\s*\(", src, re.M):
            names.add(m.group(1))
    return names


def test_library_exports_every_declared_symbol():
    names = _declared_functions()
    assert {"zero_state_bytes", "zero_init", "zero_step", "zero_gather_layer",
            "zero_destroy"} <= names
    lib = C.CDLL(A.LIB_PATH)
    for n in sorted(names):
        assert hasattr(lib, n), n


def _ledger_vs_oracle(psi, nd, stage, tensors=None, view=-1, variant=0):
    cfg = A.Config(psi, nd, stage, rank_view=view, variant=variant, tensors=tensors)
    L = A.zero_state_bytes(cfg)
    numel = [n for n, _ in tensors] if tensors else None
    assert list(L.formula_bytes) == list(Z.ledger_formula(psi, nd))
    assert list(L.exact_bytes) == list(Z.ledger_exact(psi, nd, numel))
    c = Z.comm_elements(psi, nd)
    assert list(L.comm_elements) == [c["reduce_scatter"], c["all_gather"], c["dp"], c["stage1"],
                                     c["stage2"], c["stage3"]]
    assert L.allreduce_buffer_bytes == 4 * psi
    assert L.partition_len == -(-psi // nd)
    return cfg, L


def test_ledger_matches_oracle_running_example():
    cfg, L = _ledger_vs_oracle(7_500_000_000, 64, 1, view=0)
    assert list(L.exact_bytes) == [120_000_000_000, 31_406_250_000, 16_640_625_000, 1_875_000_000]
    assert L.state_elems == 117_187_500 and L.grad_len == 117_187_500 and L.n_out == 1


def test_ledger_matches_oracle_grid():
    rng = np.random.default_rng(0)
    for psi in list(range(1, 41)) + [1000, 1_048_576, 16_777_216]:
        for nd in (1, 2, 3, 4, 7, 8, 9, 64):
            for stage in (1, 2):
                _ledger_vs_oracle(psi, nd, stage, variant=int(rng.integers(0, 2)))
    for _ in range(100):
        nd = int(rng.integers(1, 10))
        k = int(rng.integers(1, 8))
        numel = [int(x) for x in rng.integers(1, 50, size=k)]
        units = np.sort(rng.integers(0, 3, size=k))
        units = np.searchsorted(np.unique(units), units)  # contiguous from 0
        tensors = list(zip(numel, [int(u) for u in units]))
        _ledger_vs_oracle(sum(numel), nd, 3, tensors=tensors)


def test_rank_shards_match_oracle_partition():
    for psi in range(1, 41):
        for nd in range(1, 10):
            cfg = A.Config(psi, nd, 2)
            for r in range(nd):
                b, e = Z.partition(psi, nd, r)
                assert A.zero_rank_shard(cfg, r) == (b, e - b)
    rng = np.random.default_rng(1)
    for _ in range(100):
        nd = int(rng.integers(1, 10))
        numel = [int(x) for x in rng.integers(1, 30, size=rng.integers(1, 6))]
        cfg = A.Config(sum(numel), nd, 3, tensors=[(n, 0) for n in numel])
        pos = 0
        for r in range(nd):
            ln = Z.shard_len(numel, nd, r)
            assert A.zero_rank_shard(cfg, r) == (pos, ln)
            pos += ln


def test_unit_ranges_and_transient():
    wl = W.llama_2p7b()
    cfg = A.Config(wl.psi, wl.nd, 3, tensors=wl.tensors)
    L = A.zero_state_bytes(cfg)
    assert wl.psi == 2_701_560_320 and len(wl.tensors) == 291
    assert L.n_units == 34
    sizes = {}
    for n, u in wl.tensors:
        sizes[u] = sizes.get(u, 0) + n
    begin = 0
    for u in range(L.n_units):
        assert A.zero_unit_range(cfg, u) == (begin, sizes[u])
        begin += sizes[u]
    assert sizes[1] == 79_303_680
    assert L.transient_bytes == 2 * max(sizes.values()) == 2 * 81_922_560
    assert L.peak_stage3_bytes == L.exact_bytes[3] + L.transient_bytes
    gpt = W.gpt2_1p5b()
    assert gpt.psi == 1_557_611_200 and len(gpt.tensors) == 580


def test_workspace_layout():
    for variant in (0, 1, 2):
        for stage in (1, 2, 3):
            tensors = [(1000, 0), (37, 1), (5000, 1)] if stage == 3 else None
            cfg = A.Config(6037, 8, stage, variant=variant, tensors=tensors)
            L = A.zero_state_bytes(cfg)
            offs = [L.off_master[0], L.off_m[0], L.off_v[0]]
            if variant in (0, 2):
                offs += [L.off_master[1], L.off_m[1], L.off_v[1]]
                assert L.off_reduced == -1
            else:
                assert L.off_master[1] == -1 and L.off_reduced > 0
                offs.append(L.off_reduced)
            if stage == 3:
                assert L.off_shard16 > 0
            for o in offs:
                assert o % 256 == 0 and o + 4 * L.state_elems <= L.workspace_bytes
            assert len(set(offs)) == len(offs)


@pytest.mark.parametrize("kw", [
    dict(psi=0, nd=1, stage=1), dict(psi=10, nd=0, stage=1), dict(psi=10, nd=2, stage=4),
    dict(psi=10, nd=2, stage=3),  # stage 3 needs a tensor list
    dict(psi=10, nd=2, stage=2, rank_view=2), dict(psi=10, nd=2, stage=3, rank_view=0, view_outputs=2,
                                                   tensors=[(10, 0)]),  # a stage-3 rank has one output
    dict(psi=10, nd=2, stage=2, variant=7), dict(psi=10, nd=2, stage=2, tensors=[(4, 0), (5, 0)]),
    dict(psi=10, nd=2, stage=3, tensors=[(4, 1), (6, 1)]),  # units must start at 0
    dict(psi=10, nd=2, stage=3, tensors=[(4, 0), (6, 2)]),  # units must be contiguous
    dict(psi=10, nd=A.ZERO_MAX_ND + 1, stage=1),
    dict(psi=10, nd=2, stage=2, tensors=[(4, 0, 2), (6, 0)]),  # unknown tensor flag
    dict(psi=10, nd=2, stage=3, tensors=[(4, 0, -1), (6, 1)]),
])
def test_invalid_configs_rejected(kw):
    cfg = A.Config(**kw)
    with pytest.raises(A.ZeroError) as ei:
        A.zero_state_bytes(cfg)
    assert ei.value.code == A.ZERO_ERR_ARG


def test_init_validation_before_device_work():
    cfg = A.Config(1000, 4, 2)
    L = A.zero_state_bytes(cfg)
    ws = 1 << 20  # never dereferenced: validation fails first
    with pytest.raises(A.ZeroError) as ei:
        A.zero_init(cfg, ws + 8, L.workspace_bytes, ws, [ws] * 4, 0)
    assert ei.value.code == A.ZERO_ERR_ALIGN
    with pytest.raises(A.ZeroError) as ei:
        A.zero_init(cfg, ws, L.workspace_bytes - 1, ws, [ws] * 4, 0)
    assert ei.value.code == A.ZERO_ERR_WORKSPACE
    with pytest.raises(A.ZeroError) as ei:
        A.zero_init(cfg, ws, L.workspace_bytes, 0, [ws] * 4, 0)
    assert ei.value.code == A.ZERO_ERR_ARG
    with pytest.raises(A.ZeroError) as ei:
        A.zero_init(cfg, ws, L.workspace_bytes, ws, [ws, ws, ws + 2, ws], 0)
    assert ei.value.code == A.ZERO_ERR_ALIGN
    with pytest.raises(A.ZeroError) as ei:
        A.zero_init(cfg, ws, L.workspace_bytes, ws, None, 0)
    assert ei.value.code == A.ZERO_ERR_ARG


def test_error_strings():
    for code in (0, 1, -1, -2, -3, -4, -5, -6, -7):
        assert A.error_string(code) and A.error_string(code) != "unknown error code"


def test_no_decay_flag_accepted_and_layout_unchanged_in_size_order():
    """The weight-decay flag does not change the ledger; it only adds run
    table entries (a few bytes of workspace)."""
    ND = A.ZERO_TENSOR_NO_DECAY
    for stage in (1, 2, 3):
        plain = [(1000, 0), (17, 0), (3000, 1), (5, 1)]
        flagged = [(1000, 0), (17, 0, ND), (3000, 1), (5, 1, ND)]
        a = A.zero_state_bytes(A.Config(4022, 3, stage, tensors=plain))
        b = A.zero_state_bytes(A.Config(4022, 3, stage, tensors=flagged))
        assert list(a.exact_bytes) == list(b.exact_bytes)
        assert a.state_elems == b.state_elems and a.transient_bytes == b.transient_bytes
        assert b.workspace_bytes >= a.workspace_bytes
        assert b.workspace_bytes - a.workspace_bytes <= 4096


def test_bf16_precision_ledger_and_validation():
    """Without fp32 master weights K = 8 ([P3] "Why parameter count is not
    training memory"; [P2] "The Mathematics": (2 + 2 + K) Psi)."""
    BF = A.ZERO_PRECISION_BF16
    tensors = [(1000, 0), (17, 1), (3001, 1)]
    psi, nd = 4018, 3
    numel = [n for n, _ in tensors]
    P = max(e - b for b, e in (Z.partition(psi, nd, r) for r in range(nd)))
    S = max(sum(e - b for b, e in (Z.chunk(n, nd, r) for n in numel)) for r in range(nd))
    for stage in (1, 2, 3):
        L = A.zero_state_bytes(A.Config(psi, nd, stage, variant=A.ZERO_VARIANT_TWO_PASS,
                                        tensors=tensors, precision=BF))
        assert list(L.exact_bytes) == [12 * psi, 4 * psi + 8 * P, 2 * psi + 10 * P, 12 * S]
        f = list(L.formula_bytes)
        assert f == pytest.approx([12 * psi, 4 * psi + 8 * psi / nd, 2 * psi + 10 * psi / nd,
                                   12 * psi / nd], rel=1e-12)
        assert list(L.off_master) == [-1, -1] and L.off_m[0] >= 0 and L.off_v[0] >= 0
        L16 = A.zero_state_bytes(A.Config(psi, nd, stage, variant=A.ZERO_VARIANT_TWO_PASS,
                                          tensors=tensors))
        # the master array is gone from the workspace
        assert L16.workspace_bytes - L.workspace_bytes >= 4 * psi
    # both two-pass variants take bfloat16; the TMA one has the same workspace
    # plus its second run table
    Lt = A.zero_state_bytes(A.Config(psi, nd, 2, variant=A.ZERO_VARIANT_TWO_PASS_TMA, tensors=tensors,
                                     precision=BF))
    L2 = A.zero_state_bytes(A.Config(psi, nd, 2, variant=A.ZERO_VARIANT_TWO_PASS, tensors=tensors,
                                     precision=BF))
    assert list(Lt.exact_bytes) == list(L2.exact_bytes) and Lt.off_reduced > 0
    assert 0 <= Lt.workspace_bytes - L2.workspace_bytes <= 4096
    with pytest.raises(A.ZeroError) as ei:
        A.zero_state_bytes(A.Config(psi, nd, 2, precision=2))
    assert ei.value.code == A.ZERO_ERR_ARG
    # the fused step without a master rolls back from a second copy of the
    # weights, the last replica: emulated stage 1/2 ranks with Nd >= 2 only;
    # it keeps two m/v buffers and no reduced-gradient scratch
    for variant in (A.ZERO_VARIANT_FUSED, A.ZERO_VARIANT_FUSED_TMA):
        for stage in (1, 2):
            Lf = A.zero_state_bytes(A.Config(psi, nd, stage, variant=variant, tensors=tensors, precision=BF))
            assert list(Lf.off_master) == [-1, -1] and min(Lf.off_m) >= 0 and min(Lf.off_v) >= 0
            assert Lf.off_reduced < 0
            assert list(Lf.exact_bytes) == list(L2.exact_bytes)
        for bad in (dict(nd=1, stage=2), dict(nd=nd, stage=3), dict(nd=nd, stage=1, rank_view=0)):
            with pytest.raises(A.ZeroError) as ei:
                A.zero_state_bytes(A.Config(psi, bad["nd"], bad["stage"], rank_view=bad.get("rank_view", -1),
                                            variant=variant, tensors=tensors, precision=BF))
            assert ei.value.code == A.ZERO_ERR_ARG
    with pytest.raises(A.ZeroError):
        A.zero_offload_bytes(A.Config(psi, nd, 2, variant=A.ZERO_VARIANT_TWO_PASS, precision=BF))
