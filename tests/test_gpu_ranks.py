"""The per-rank step of a real Nd-rank job (single-rank view with
view_outputs = nd; zero_flag_words), emulated on one GPU: Nd handles, one per
rank, share the ranks' gradient buffers and replica buffers exactly as peer
mappings would; each handle reads its partition of every rank's gradient and
writes its partition into every replica; between launch and commit the
handles' flag words are MAX-reduced (what an NCCL all-reduce does across
processes). The result must equal the plain data-parallel definition ([P2]
"The Breakthrough": ZeRO leaves the training math untouched).

The handles run one after another on one stream here: nothing waits on
another rank's kernel, so no emulation of concurrent ranks is needed.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

from oracle import zero_ref as Z
from zero_partitioned_mixed_02_b200 import _abi as A
from zero_partitioned_mixed_02_b200 import synth as S
from zero_partitioned_mixed_02_b200.distributed import flag_words

from gpu_common import GuardedF16, compare_f16, compare_f32, hyper

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a GPU", allow_module_level=True)


def _job(psi, nd, stage, variant, steps, inject=(), precision=A.ZERO_PRECISION_FP16, tensors=None):
    s = torch.cuda.current_stream()
    w0 = S.host_f32(psi, 0, S.key(4, S.STREAM_MASTER, 0, 0), S.uniform(-1.0, 1.0))
    m_init = torch.from_numpy(w0.copy()).cuda()
    reps = [GuardedF16(psi) for _ in range(nd)]
    G = [torch.empty(psi, dtype=torch.int16, device="cuda") for _ in range(nd)]
    handles, wss, parts = [], [], []
    for r in range(nd):
        cfg = A.Config(psi, nd, stage, rank_view=r, variant=variant, tensors=tensors, precision=precision,
                       view_outputs=nd)
        L = A.zero_state_bytes(cfg)
        assert L.n_out == nd
        b, e = Z.partition(psi, nd, r)
        ws = torch.empty(L.workspace_bytes, dtype=torch.uint8, device="cuda")
        h = A.zero_init(cfg, ws.data_ptr(), L.workspace_bytes, m_init.data_ptr() + 4 * b,
                        [x.ptr() for x in reps], s.cuda_stream)
        handles.append(h)
        wss.append(ws)
        parts.append((b, e))
    bf16 = precision == A.ZERO_PRECISION_BF16
    mask = Z.decay_mask([t[0] for t in tensors], [bool(t[2]) if len(t) > 2 else False for t in tensors]) \
        if tensors else None
    w, m, v = w0.copy(), np.zeros(psi, np.float32), np.zeros(psi, np.float32)
    p = Z.bf16_from_f32(w) if bf16 else Z.f16_from_f32(w)
    t = 0
    hp = dict(lr=1e-2, weight_decay=0.05)
    skips = []
    for step in range(steps):
        if bf16:
            gs = [Z.bf16_from_f32(S.host_f32(psi, 0, S.key(4, S.STREAM_GRAD, step, k), S.normal(1e-3, 1.0)))
                  for k in range(nd)]
        else:
            gs = [S.host_f16_bits(psi, 0, S.key(4, S.STREAM_GRAD, step, k), S.normal(1e-3, 1024.0))
                  for k in range(nd)]
        for (st, k, i, bits) in inject:
            if st == step:
                gs[k][i] = bits
        for k in range(nd):
            G[k].copy_(torch.from_numpy(gs[k].view(np.int16)))
        scale = 1.0 if bf16 else 1024.0
        for r, h in enumerate(handles):
            b, _ = parts[r]
            A.zero_step_launch(h, [g.data_ptr() + 2 * b for g in G], scale, hyper(**hp), s.cuda_stream)
        # the flag all-reduce (MAX) of a real job
        words = [flag_words(h) for h in handles]
        agreed = torch.stack(words).max(dim=0).values
        for x in words:
            x.copy_(agreed)
        rcs = [A.zero_step_commit(h, s.cuda_stream) for h in handles]
        assert len(set(rcs)) == 1
        if bf16:
            sk, t = Z.bf16_step(gs, p, m, v, scale, Z.hyper(**hp), t, decay=mask)
        else:
            sk, t = Z.dp_step(gs, w, m, v, p, scale, Z.hyper(**hp), t, decay=mask)
        assert (rcs[0] == A.ZERO_SKIPPED) == sk
        skips.append(sk)
        # every rank's partition of the state, every replica
        for r, h in enumerate(handles):
            b, e = parts[r]
            wp, mp, vp, tt = A.zero_current_state(h)
            assert tt == t
            base = wss[r].data_ptr()
            n = e - b
            if n:
                gm = wss[r][mp - base: mp - base + 4 * n].view(torch.float32).cpu().numpy()
                compare_f32(gm, m[b:e], f"rank {r} m, step {step}")
                if not bf16:
                    gw = wss[r][wp - base: wp - base + 4 * n].view(torch.float32).cpu().numpy()
                    compare_f32(gw, w[b:e], f"rank {r} master, step {step}")
        for k, x in enumerate(reps):
            compare_f16(x.bits(), p, f"replica {k}, step {step}")
            assert x.guards_intact()
    for h in handles:
        A.zero_destroy(h)
    return skips


VARIANTS = [A.ZERO_VARIANT_FUSED, A.ZERO_VARIANT_TWO_PASS, A.ZERO_VARIANT_FUSED_TMA, A.ZERO_VARIANT_TWO_PASS_TMA]


@pytest.mark.parametrize("variant", VARIANTS)
@pytest.mark.parametrize("nd", [1, 2, 4, 8])
def test_ranks_as_handles(nd, variant):
    # partitions of 8000 elements (16-byte aligned slices), the last one
    # nd - 1 elements short
    psi = 8000 * nd - (nd - 1)
    assert Z.partition(psi, nd, nd - 1)[0] == 8000 * (nd - 1)
    assert _job(psi, nd, 2, variant, 3, inject=[(1, nd - 1, 0, 0x7C00)]) == [False, True, False]


@pytest.mark.parametrize("variant", [A.ZERO_VARIANT_TWO_PASS, A.ZERO_VARIANT_TWO_PASS_TMA])
def test_ranks_as_handles_bf16_with_excluded_tensor(variant):
    nd = 4
    psi = 8000 * nd
    tensors = [(20_000, 0), (psi - 20_000, 0, A.ZERO_TENSOR_NO_DECAY)]
    assert _job(psi, nd, 1, variant, 2, precision=A.ZERO_PRECISION_BF16, tensors=tensors) == [False, False]


def test_view_outputs_validation():
    for kw in (dict(rank_view=-1, view_outputs=4), dict(rank_view=0, view_outputs=3)):
        with pytest.raises(A.ZeroError):
            A.zero_state_bytes(A.Config(1000, 4, 2, **kw))


def test_rank_handles_refuse_asynchronous_steps():
    nd, psi = 4, 4 * 8000
    cfg = A.Config(psi, nd, 2, rank_view=1, view_outputs=nd)
    L = A.zero_state_bytes(cfg)
    ws = torch.empty(L.workspace_bytes, dtype=torch.uint8, device="cuda")
    m0 = torch.zeros(8000, dtype=torch.float32, device="cuda")
    reps = [torch.zeros(psi, dtype=torch.int16, device="cuda") for _ in range(nd)]
    G = [torch.zeros(8000, dtype=torch.int16, device="cuda") for _ in range(nd)]
    s = torch.cuda.current_stream().cuda_stream
    h = A.zero_init(cfg, ws.data_ptr(), L.workspace_bytes, m0.data_ptr(), [r.data_ptr() for r in reps], s)
    with pytest.raises(A.ZeroError) as ei:
        A.zero_async_begin(h, [g.data_ptr() for g in G], A.zero_scaler(1.0, 2.0, 0.5, 10), 0.9, 0.999, s)
    assert ei.value.code == A.ZERO_ERR_ARG
    A.zero_destroy(h)


# stage 3: rank r of a real job keeps shard r; layer units are gathered from
# the Nd ranks' shards (zero_gather_layer_ranks). Tensor lists: chunks in
# 16-byte phase with runs of several gather tiles, and chunks out of phase
# with a ragged tail.
SHAPES3 = {
    "aligned": [(8192, 0), (4096, 0), (65536, 1), (64, 1), (16384, 2)],
    "ragged": [(4000, 0), (1601, 0), (40001, 1), (2048, 1), (777, 2), (5000, 3)],
}


def _shards(x, numel, nd, r):
    """Rank r's chunks of every tensor, concatenated (the oracle's shard)."""
    out, off = [], 0
    for n in numel:
        b, e = Z.chunk(n, nd, r)
        out.append(x[off + b: off + e])
        off += n
    return np.concatenate(out) if out else x[:0]


@pytest.mark.parametrize("variant", VARIANTS)
@pytest.mark.parametrize("nd", [2, 4])
@pytest.mark.parametrize("shape", list(SHAPES3))
def test_stage3_ranks_as_handles(shape, nd, variant):
    tensors = SHAPES3[shape]
    numel = [t[0] for t in tensors]
    unit_of = [t[1] for t in tensors]
    n_units = unit_of[-1] + 1
    psi = sum(numel)
    s = torch.cuda.current_stream()
    w0 = S.host_f32(psi, 0, S.key(5, S.STREAM_MASTER, 0, 0), S.uniform(-1.0, 1.0))
    m_init = torch.from_numpy(w0.copy()).cuda()
    G = [torch.empty(psi, dtype=torch.int16, device="cuda") for _ in range(nd)]
    handles, wss, Ls = [], [], []
    for r in range(nd):
        cfg = A.Config(psi, nd, 3, rank_view=r, variant=variant, tensors=tensors)
        L = A.zero_state_bytes(cfg)
        assert L.state_elems == Z.shard_len(numel, nd, r) and L.grad_len == psi
        ws = torch.empty(L.workspace_bytes, dtype=torch.uint8, device="cuda")
        handles.append(A.zero_init(cfg, ws.data_ptr(), L.workspace_bytes, m_init.data_ptr(), None, s.cuda_stream))
        wss.append(ws)
        Ls.append(L)
    shard_ptrs = [wss[k].data_ptr() + Ls[k].off_shard16 for k in range(nd)]
    w_sh = [_shards(w0, numel, nd, r).copy() for r in range(nd)]
    m_sh = [np.zeros_like(x) for x in w_sh]
    v_sh = [np.zeros_like(x) for x in w_sh]
    p_sh = [Z.f16_from_f32(x) for x in w_sh]
    hp = dict(lr=1e-2, weight_decay=0.05)
    t = 0
    skips = []
    for step in range(3):
        gs = [S.host_f16_bits(psi, 0, S.key(5, S.STREAM_GRAD, step, k), S.normal(1e-3, 1024.0))
              for k in range(nd)]
        if step == 1:
            gs[nd - 1][psi - 1] = 0x7E00  # a NaN on the last rank, in the last rank's last chunk
        for k in range(nd):
            G[k].copy_(torch.from_numpy(gs[k].view(np.int16)))
        for h in handles:
            A.zero_step_launch(h, [g.data_ptr() for g in G], 1024.0, hyper(**hp), s.cuda_stream)
        words = [flag_words(h) for h in handles]
        agreed = torch.stack(words).max(dim=0).values
        for x in words:
            x.copy_(agreed)
        rcs = [A.zero_step_commit(h, s.cuda_stream) for h in handles]
        assert len(set(rcs)) == 1
        sk, t = Z.zero3_step(numel, gs, w_sh, m_sh, v_sh, p_sh, 1024.0, Z.hyper(**hp), t)
        assert (rcs[0] == A.ZERO_SKIPPED) == sk
        skips.append(sk)
        for r, h in enumerate(handles):
            wp, mp, _, tt = A.zero_current_state(h)
            assert tt == t
            n = Ls[r].state_elems
            base = wss[r].data_ptr()
            compare_f32(wss[r][wp - base: wp - base + 4 * n].view(torch.float32).cpu().numpy(), w_sh[r],
                        f"rank {r} master shard, step {step}")
            compare_f32(wss[r][mp - base: mp - base + 4 * n].view(torch.float32).cpu().numpy(), m_sh[r],
                        f"rank {r} m shard, step {step}")
            o = Ls[r].off_shard16
            compare_f16(wss[r][o: o + 2 * n].view(torch.int16).cpu().numpy().view(np.uint16), p_sh[r],
                        f"rank {r} fp16 shard, step {step}")
        for u in range(n_units):
            want = Z.zero3_gather(numel, unit_of, nd, u, p_sh)
            out = GuardedF16(len(want))
            A.zero_gather_layer_ranks(handles[u % nd], u, shard_ptrs, out.ptr(), s.cuda_stream)
            compare_f16(out.bits(), want, f"unit {u} gathered by rank {u % nd}, step {step}")
            assert out.guards_intact()
        torch.cuda.synchronize()
    assert skips == [False, True, False]
    # the errors a rank's gather reports (before any launch)
    spare = GuardedF16(max(numel))
    with pytest.raises(A.ZeroError) as ei:
        A.zero_gather_layer(handles[0], 0, spare.ptr(), s.cuda_stream)
    assert ei.value.code == A.ZERO_ERR_ARG
    with pytest.raises(A.ZeroError) as ei:
        A.zero_gather_layer_ranks(handles[0], n_units, shard_ptrs, spare.ptr(), s.cuda_stream)
    assert ei.value.code == A.ZERO_ERR_ARG
    with pytest.raises(A.ZeroError) as ei:
        A.zero_gather_layer_ranks(handles[0], 0, [p + 2 for p in shard_ptrs], spare.ptr(), s.cuda_stream)
    assert ei.value.code == A.ZERO_ERR_ALIGN
    torch.cuda.synchronize()
    assert spare.guards_intact()
    for h in handles:
        A.zero_destroy(h)


def test_stage3_rank_refuses_asynchronous_steps():
    tensors = SHAPES3["aligned"]
    psi = sum(t[0] for t in tensors)
    cfg = A.Config(psi, 2, 3, rank_view=1, tensors=tensors)
    L = A.zero_state_bytes(cfg)
    ws = torch.empty(L.workspace_bytes, dtype=torch.uint8, device="cuda")
    m0 = torch.zeros(psi, dtype=torch.float32, device="cuda")
    G = [torch.zeros(psi, dtype=torch.int16, device="cuda") for _ in range(2)]
    s = torch.cuda.current_stream().cuda_stream
    h = A.zero_init(cfg, ws.data_ptr(), L.workspace_bytes, m0.data_ptr(), None, s)
    with pytest.raises(A.ZeroError) as ei:
        A.zero_async_begin(h, [g.data_ptr() for g in G], A.zero_scaler(1.0, 2.0, 0.5, 10), 0.9, 0.999, s)
    assert ei.value.code == A.ZERO_ERR_ARG
    A.zero_destroy(h)
