"""The three large workloads at full size, in the launch configuration the
benchmark times, checked against the oracle on sampled outputs (the oracle
computes each sampled element's whole trajectory from the same generated
inputs) and by properties that hold at any size:

  GPT-2 1.5B-shaped list, Psi = 1,557,611,200, Nd = 8, stage 2, AdamW, 5 steps
  Psi = 7.5e9, Nd = 64, rank-0 view (P = 117,187,500), stage 1, 5 steps
  Llama 2.7B-shaped list, Psi = 2,701,560,320, Nd = 8, stage 3, 3 steps, with
  the layer gathers forward then reverse after every step

Samples: every partition / tensor / chunk boundary (and its neighbours), the
first and last elements, plus 20,000 uniform draws.
"""
from __future__ import annotations

import gc

import numpy as np
import pytest
import torch

from oracle import zero_ref as Z
from zero_partitioned_mixed_02_b200 import _abi as A
from zero_partitioned_mixed_02_b200 import synth as S
from zero_partitioned_mixed_02_b200.synth import workloads as W

from gpu_common import compare_f16, compare_f32, host_f32, host_u16, hyper

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a GPU", allow_module_level=True)

SENT = np.int16(0x5A5A)


def _samples(wl, b0, e0, rng):
    pts = [b0, b0 + 1, b0 + 7, b0 + 8, e0 - 9, e0 - 8, e0 - 1]
    if wl.rank_view < 0:
        for r in range(wl.nd):
            b, _ = Z.partition(wl.psi, wl.nd, r)
            pts += [b - 1, b, b + 1]
    if wl.tensors:
        offs = np.concatenate([[0], np.cumsum([n for n, _ in wl.tensors])])
        for t, (n, _) in enumerate(wl.tensors):
            pts += [offs[t] - 1, offs[t], offs[t] + 1]
            if wl.stage == 3:
                for r in range(wl.nd):
                    cb, ce = Z.chunk(n, wl.nd, r)
                    pts += [offs[t] + cb - 1, offs[t] + cb, offs[t] + ce - 1]
    pts += list(rng.integers(b0, e0, size=20_000))
    idx = np.unique(np.array(pts, dtype=np.int64))
    return idx[(idx >= b0) & (idx < e0)]


def _stage3_state_index(wl, idx):
    numel = np.array([n for n, _ in wl.tensors], dtype=np.int64)
    offs = np.concatenate([[0], np.cumsum(numel)])
    nd = wl.nd
    chunk_len = np.array([[Z.chunk(int(n), nd, r)[1] - Z.chunk(int(n), nd, r)[0] for n in numel]
                          for r in range(nd)], dtype=np.int64)
    shard_begin = np.concatenate([[0], np.cumsum(chunk_len.sum(axis=1))])[:nd]
    before = np.concatenate([np.zeros((nd, 1), np.int64), np.cumsum(chunk_len, axis=1)], axis=1)
    t = np.searchsorted(offs, idx, side="right") - 1
    j = idx - offs[t]
    c = -(-numel[t] // nd)
    r = j // c
    q = j - r * c
    return shard_begin[r] + before[r, t] + q


def _run(wl: W.Workload, variant: int):
    rng = np.random.default_rng(123)
    cfg = A.Config(wl.psi, wl.nd, wl.stage, rank_view=wl.rank_view, variant=variant,
                   tensors=wl.tensors)
    L = A.zero_state_bytes(cfg)
    b0, e0 = (Z.partition(wl.psi, wl.nd, wl.rank_view) if wl.rank_view >= 0 else (0, wl.psi))
    n_own = e0 - b0
    st = torch.cuda.current_stream()
    s = st.cuda_stream
    ws = torch.empty(L.workspace_bytes, dtype=torch.uint8, device="cuda")
    m_init = torch.empty(n_own, dtype=torch.float32, device="cuda")
    kmaster = S.key(wl.seed, S.STREAM_MASTER, 0, 0)
    S.fill_f32(m_init.data_ptr(), n_own, b0, kmaster, wl.master, s)
    bufs = []
    if wl.stage <= 2:
        nb = wl.nd if wl.rank_view < 0 else 1
        bufs = [torch.full((wl.psi,), SENT, dtype=torch.int16, device="cuda") for _ in range(nb)]
    grads = [torch.empty(n_own, dtype=torch.int16, device="cuda") for _ in range(wl.nd)]
    h = A.zero_init(cfg, ws.data_ptr(), L.workspace_bytes, m_init.data_ptr(),
                    [b.data_ptr() for b in bufs] if bufs else None, s)
    del m_init
    idx = _samples(wl, b0, e0, rng)
    w_o = S.host_f32_at(idx, kmaster, wl.master)
    m_o = np.zeros_like(w_o)
    v_o = np.zeros_like(w_o)
    p_o = Z.f16_from_f32(w_o)
    t_o = 0
    hp_o = Z.hyper(**wl.hyper)
    units_out = None
    for step in range(wl.steps):
        for k in range(wl.nd):
            S.fill_f16(grads[k].data_ptr(), n_own, b0, S.key(wl.seed, S.STREAM_GRAD, step, k),
                       wl.grad, s)
        rc = A.zero_step(h, [g.data_ptr() for g in grads], wl.loss_scale, hyper(**wl.hyper), s)
        gs = [S.host_f16_bits_at(idx, S.key(wl.seed, S.STREAM_GRAD, step, k), wl.grad)
              for k in range(wl.nd)]
        sk, t_o = Z.dp_step(gs, w_o, m_o, v_o, p_o, wl.loss_scale, hp_o, t_o)
        assert rc == A.ZERO_OK and not sk
        if wl.stage == 3:
            # the layer gathers of a training step: forward 0..U-1, backward U-1..0
            max_unit = max(A.zero_unit_range(cfg, u)[1] for u in range(L.n_units))
            out = torch.empty(max_unit, dtype=torch.int16, device="cuda")
            order = list(range(L.n_units)) + list(reversed(range(L.n_units)))
            units_out = {}
            for u in order:
                A.zero_gather_layer(h, u, out.data_ptr(), s)
                fb, cnt = A.zero_unit_range(cfg, u)
                sel = idx[(idx >= fb) & (idx < fb + cnt)]
                units_out[u] = (sel, host_u16(out[torch.from_numpy(sel - fb).cuda()]))
            del out
    wp, mp, vp, t = A.zero_current_state(h)
    assert t == t_o == wl.steps
    base = ws.data_ptr()
    n = L.state_elems

    def view(p):
        return ws[p - base: p - base + 4 * n].view(torch.float32)

    w_g, m_g, v_g = view(wp), view(mp), view(vp)
    if wl.stage == 3:
        sidx = _stage3_state_index(wl, idx)
    else:
        sidx = idx - b0
    sel = torch.from_numpy(sidx).cuda()
    compare_f32(host_f32(w_g[sel]), w_o, "master (sampled)")
    compare_f32(host_f32(m_g[sel]), m_o, "m (sampled)")
    compare_f32(host_f32(v_g[sel]), v_o, "v (sampled)")
    isel = torch.from_numpy(idx).cuda()
    half_master = w_g.half().view(torch.int16)  # torch's own round-to-nearest-even
    if wl.stage <= 2:
        for k, b in enumerate(bufs):
            compare_f16(host_u16(b[isel]), p_o, f"replica {k} (sampled)")
        part = bufs[0][b0:e0]
        assert torch.equal(part, half_master), "fp16 params != fp16(master) somewhere"
        for b in bufs[1:]:
            assert torch.equal(b, bufs[0]), "replicas differ"
        if wl.rank_view >= 0:
            assert bool((bufs[0][:b0] == SENT).all()) and bool((bufs[0][e0:] == SENT).all())
    else:
        sh = ws[L.off_shard16: L.off_shard16 + 2 * n].view(torch.int16)
        compare_f16(host_u16(sh[sel]), p_o, "fp16 shard (sampled)")
        assert torch.equal(sh, half_master), "fp16 shard != fp16(master) somewhere"
        for u, (us, got) in units_out.items():
            pos = np.searchsorted(idx, us)
            compare_f16(got, p_o[pos], f"gathered unit {u} (sampled)")
    A.zero_destroy(h)
    del ws, bufs, grads, w_g, m_g, v_g, half_master
    gc.collect()
    torch.cuda.empty_cache()


@pytest.mark.parametrize("variant", [A.ZERO_VARIANT_FUSED, A.ZERO_VARIANT_TWO_PASS, A.ZERO_VARIANT_FUSED_TMA,
                                     A.ZERO_VARIANT_TWO_PASS_TMA])
def test_gpt2_1p5b_stage2(variant):
    _run(W.gpt2_1p5b(), variant)


@pytest.mark.parametrize("variant", [A.ZERO_VARIANT_FUSED, A.ZERO_VARIANT_TWO_PASS, A.ZERO_VARIANT_FUSED_TMA,
                                     A.ZERO_VARIANT_TWO_PASS_TMA])
def test_running_example_7p5b_rank_view(variant):
    _run(W.running_example_7p5b(), variant)


@pytest.mark.parametrize("variant", [A.ZERO_VARIANT_FUSED, A.ZERO_VARIANT_TWO_PASS, A.ZERO_VARIANT_FUSED_TMA,
                                     A.ZERO_VARIANT_TWO_PASS_TMA])
def test_llama_2p7b_stage3(variant):
    _run(W.llama_2p7b(), variant)


def _bf16_grad(k, step, wl, b0, n_own, out, s):
    """The generator's binary32 gradient rounded to bfloat16 on the device,
    the way the benchmark makes it."""
    tmp = torch.empty(n_own, dtype=torch.float32, device="cuda")
    S.fill_f32(tmp.data_ptr(), n_own, b0, S.key(wl.seed, S.STREAM_GRAD, step, k), wl.grad, s)
    out.copy_(tmp.to(torch.bfloat16).view(torch.int16))


@pytest.mark.parametrize("variant", [A.ZERO_VARIANT_TWO_PASS, A.ZERO_VARIANT_TWO_PASS_TMA])
def test_gpt2_1p5b_bf16_without_master(variant):
    """The bfloat16 step without master weights at full size (bench
    --precision bf16): sampled m, v and parameters against the oracle's
    zr_bf16_step, every replica identical."""
    wl = W.gpt2_1p5b()
    rng = np.random.default_rng(321)
    cfg = A.Config(wl.psi, wl.nd, wl.stage, variant=variant, tensors=wl.tensors,
                   precision=A.ZERO_PRECISION_BF16)
    L = A.zero_state_bytes(cfg)
    n = wl.psi
    s = torch.cuda.current_stream().cuda_stream
    ws = torch.empty(L.workspace_bytes, dtype=torch.uint8, device="cuda")
    kmaster = S.key(wl.seed, S.STREAM_MASTER, 0, 0)
    m_init = torch.empty(n, dtype=torch.float32, device="cuda")
    S.fill_f32(m_init.data_ptr(), n, 0, kmaster, wl.master, s)
    bufs = [torch.full((n,), SENT, dtype=torch.int16, device="cuda") for _ in range(wl.nd)]
    grads = [torch.empty(n, dtype=torch.int16, device="cuda") for _ in range(wl.nd)]
    h = A.zero_init(cfg, ws.data_ptr(), L.workspace_bytes, m_init.data_ptr(), [b.data_ptr() for b in bufs], s)
    del m_init
    idx = _samples(wl, 0, n, rng)
    w16 = Z.bf16_from_f32(S.host_f32_at(idx, kmaster, wl.master))
    m_o, v_o, t_o = np.zeros(idx.size, np.float32), np.zeros(idx.size, np.float32), 0
    steps = 3
    for step in range(steps):
        for k in range(wl.nd):
            _bf16_grad(k, step, wl, 0, n, grads[k], s)
        rc = A.zero_step(h, [g.data_ptr() for g in grads], wl.loss_scale, hyper(**wl.hyper), s)
        gs = [Z.bf16_from_f32(S.host_f32_at(idx, S.key(wl.seed, S.STREAM_GRAD, step, k), wl.grad))
              for k in range(wl.nd)]
        sk, t_o = Z.bf16_step(gs, w16, m_o, v_o, wl.loss_scale, Z.hyper(**wl.hyper), t_o)
        assert rc == A.ZERO_OK and not sk
    wp, mp, vp, t = A.zero_current_state(h)
    assert wp is None and t == t_o == steps
    base = ws.data_ptr()
    sel = torch.from_numpy(idx).cuda()
    compare_f32(host_f32(ws[mp - base: mp - base + 4 * n].view(torch.float32)[sel]), m_o, "m (sampled)")
    compare_f32(host_f32(ws[vp - base: vp - base + 4 * n].view(torch.float32)[sel]), v_o, "v (sampled)")
    for k, b in enumerate(bufs):
        compare_f16(host_u16(b[sel]), w16, f"bf16 replica {k} (sampled)")
    for b in bufs[1:]:
        assert torch.equal(b, bufs[0]), "replicas differ"
    A.zero_destroy(h)
    del ws, bufs, grads
    gc.collect()
    torch.cuda.empty_cache()


def test_gpt2_1p5b_offload():
    """The offloaded step at full size with the default chunk and all host
    threads (bench --offload): the host master, m, v sampled against the
    oracle, every replica identical and equal to fp16 of the host master."""
    import os

    wl = W.gpt2_1p5b()
    rng = np.random.default_rng(654)
    cfg = A.Config(wl.psi, wl.nd, wl.stage, tensors=wl.tensors)
    L = A.zero_offload_bytes(cfg, 0)
    n = wl.psi
    s = torch.cuda.current_stream().cuda_stream
    kmaster = S.key(wl.seed, S.STREAM_MASTER, 0, 0)
    m_dev = torch.empty(n, dtype=torch.float32, device="cuda")
    S.fill_f32(m_dev.data_ptr(), n, 0, kmaster, wl.master, s)
    master_init = m_dev.cpu().numpy()
    del m_dev
    state = np.empty(3 * n, np.float32)
    dws = torch.empty(L.device_bytes, dtype=torch.uint8, device="cuda")
    staging = torch.empty(L.host_staging_bytes, dtype=torch.uint8, pin_memory=True)
    bufs = [torch.full((n,), SENT, dtype=torch.int16, device="cuda") for _ in range(wl.nd)]
    grads = [torch.empty(n, dtype=torch.int16, device="cuda") for _ in range(wl.nd)]
    threads = len(os.sched_getaffinity(0))
    h = A.zero_offload_init(cfg, 0, dws.data_ptr(), L.device_bytes, staging.data_ptr(), L.host_staging_bytes,
                            state.ctypes.data, master_init.ctypes.data, [b.data_ptr() for b in bufs],
                            threads, s)
    del master_init
    idx = _samples(wl, 0, n, rng)
    w_o = S.host_f32_at(idx, kmaster, wl.master)
    m_o, v_o, p_o, t_o = np.zeros_like(w_o), np.zeros_like(w_o), Z.f16_from_f32(w_o), 0
    steps = 2
    for step in range(steps):
        for k in range(wl.nd):
            S.fill_f16(grads[k].data_ptr(), n, 0, S.key(wl.seed, S.STREAM_GRAD, step, k), wl.grad, s)
        rc = A.zero_offload_step(h, [g.data_ptr() for g in grads], wl.loss_scale, hyper(**wl.hyper), s)
        gs = [S.host_f16_bits_at(idx, S.key(wl.seed, S.STREAM_GRAD, step, k), wl.grad) for k in range(wl.nd)]
        sk, t_o = Z.dp_step(gs, w_o, m_o, v_o, p_o, wl.loss_scale, Z.hyper(**wl.hyper), t_o)
        assert rc == A.ZERO_OK and not sk
    torch.cuda.synchronize()
    assert A.zero_offload_state(h)[3] == t_o == steps
    compare_f32(state[idx], w_o, "host master (sampled)")
    compare_f32(state[n + idx], m_o, "host m (sampled)")
    compare_f32(state[2 * n + idx], v_o, "host v (sampled)")
    sel = torch.from_numpy(idx).cuda()
    for k, b in enumerate(bufs):
        compare_f16(host_u16(b[sel]), p_o, f"replica {k} (sampled)")
    for b in bufs[1:]:
        assert torch.equal(b, bufs[0]), "replicas differ"
    half_master = torch.from_numpy(state[:n]).cuda().half().view(torch.int16)
    assert torch.equal(bufs[0], half_master), "fp16 params != fp16(host master) somewhere"
    A.zero_offload_destroy(h)
    del dws, bufs, grads, half_master, state
    gc.collect()
    torch.cuda.empty_cache()
