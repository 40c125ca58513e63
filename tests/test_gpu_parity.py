"""GPU vs oracle, element by element, through the C ABI.

Sizes the oracle finishes in seconds: a grid of tiny and ragged cases (every
stage and variant, Nd 1..9, Psi from 1 to a few thousand with ragged tails and
empty partitions, stage-3 tensor lists with odd sizes), the single-rank view
with out-of-phase partitions, overflow skips (inf, -inf, NaN, an unscale that
overflows) injected where the injecting rank does not own the element, and
the two small workloads in full (Psi = 1,048,576, Nd = 4, stage 2;
Psi = 16,777,216, Nd = 8, stage 1, precision stress with a skip).
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

from oracle import zero_ref as Z
from zero_partitioned_mixed_02_b200 import _abi as A
from zero_partitioned_mixed_02_b200 import synth as S
from zero_partitioned_mixed_02_b200.synth import workloads as W

from gpu_common import (GuardedF16, GuardedWorkspace, SENTINEL16, compare_f16, compare_f32,
                        dev_u16, hyper, state_offsets)

pytestmark = pytest.mark.gpu

VARIANTS = [A.ZERO_VARIANT_FUSED, A.ZERO_VARIANT_TWO_PASS, A.ZERO_VARIANT_FUSED_TMA,
            A.ZERO_VARIANT_TWO_PASS_TMA]
TMA_VARIANTS = [A.ZERO_VARIANT_FUSED_TMA, A.ZERO_VARIANT_TWO_PASS_TMA]

if not torch.cuda.is_available():  # collected on CPU machines, never run there
    pytest.skip("needs a GPU", allow_module_level=True)


def _tensor_list(rng, psi, n_max=6):
    k = int(rng.integers(1, min(n_max, psi) + 1))
    cuts = np.sort(rng.choice(np.arange(1, psi), size=k - 1, replace=False)) if k > 1 else []
    sizes = np.diff(np.concatenate([[0], cuts, [psi]])).astype(int)
    units = np.sort(rng.integers(0, 3, size=k))
    units = np.searchsorted(np.unique(units), units)
    return [(int(n), int(u)) for n, u in zip(sizes, units)]


class Case:
    """One configuration driven step by step on the GPU and in the oracle."""

    def __init__(self, psi, nd, stage, variant, *, tensors=None, view=-1, loss_scale=1024.0,
                 hp=None, grad_dist=None, master_dist=None, seed=0):
        self.psi, self.nd, self.stage, self.variant, self.view = psi, nd, stage, variant, view
        self.tensors = tensors
        self.numel = [t[0] for t in tensors] if tensors else [psi]
        self.units = [t[1] for t in tensors] if tensors else [0]
        self.loss_scale = loss_scale
        self.hp = hp or {}
        self.grad_dist = grad_dist or S.normal(1e-3, loss_scale)
        self.master_dist = master_dist or S.uniform(-0.1, 0.1)
        self.seed = seed
        self.cfg = A.Config(psi, nd, stage, rank_view=view, variant=variant, tensors=tensors)
        self.L = A.zero_state_bytes(self.cfg)
        if view >= 0:
            self.b0, self.e0 = Z.partition(psi, nd, view)
        else:
            self.b0, self.e0 = 0, psi
        n_own = self.e0 - self.b0
        self.master0 = S.host_f32(n_own, self.b0, S.key(seed, S.STREAM_MASTER, 0, 0),
                                  self.master_dist)
        # ---- GPU ----
        self.ws = GuardedWorkspace(self.L.workspace_bytes)
        self.m_init = torch.from_numpy(self.master0.copy()).cuda()
        self.bufs = []
        ptrs = None
        if stage <= 2:
            self.bufs = [GuardedF16(psi) for _ in range(nd if view < 0 else 1)]
            ptrs = [b.ptr() for b in self.bufs]
        self.stream = torch.cuda.current_stream().cuda_stream
        self.h = A.zero_init(self.cfg, self.ws.ptr(), self.L.workspace_bytes,
                             self.m_init.data_ptr(), ptrs, self.stream)
        self.g_dev = [torch.empty(max(n_own, 1), dtype=torch.int16, device="cuda")
                      for _ in range(nd)]
        # ---- oracle ----
        self.t = 0
        if stage <= 2 and view < 0:
            parts = [Z.partition(psi, nd, r) for r in range(nd)]
            self.w_sh = [self.master0[b:e].copy() for b, e in parts]
            self.m_sh = [np.zeros(e - b, np.float32) for b, e in parts]
            self.v_sh = [np.zeros(e - b, np.float32) for b, e in parts]
            self.reps = [Z.f16_from_f32(self.master0) for _ in range(nd)]
        elif view >= 0:
            self.w = self.master0.copy()
            self.m = np.zeros(n_own, np.float32)
            self.v = np.zeros(n_own, np.float32)
            self.p16 = Z.f16_from_f32(self.w)
        else:
            offs = np.concatenate([[0], np.cumsum(self.numel)])
            self.w_sh = []
            for r in range(nd):
                pieces = [self.master0[offs[t] + b: offs[t] + e]
                          for t, n in enumerate(self.numel) for b, e in [Z.chunk(n, nd, r)]]
                self.w_sh.append(np.concatenate(pieces).astype(np.float32))
            self.m_sh = [np.zeros_like(x) for x in self.w_sh]
            self.v_sh = [np.zeros_like(x) for x in self.w_sh]
            self.p_sh = [Z.f16_from_f32(x) for x in self.w_sh]

    def grads(self, step):
        n = self.e0 - self.b0
        return [S.host_f16_bits(n, self.b0, S.key(self.seed, S.STREAM_GRAD, step, k),
                                self.grad_dist) for k in range(self.nd)]

    def upload(self, gs):
        n = self.e0 - self.b0
        for k in range(self.nd):
            if n:
                self.g_dev[k][:n].copy_(torch.from_numpy(gs[k].view(np.int16)))

    def oracle_step(self, gs, loss_scale):
        hp = Z.hyper(**self.hp)
        if self.stage <= 2 and self.view < 0:
            sk, self.t = Z.zero12_step(self.psi, gs, self.w_sh, self.m_sh, self.v_sh, self.reps,
                                       loss_scale, hp, self.t)
        elif self.view >= 0:
            sk, self.t = Z.dp_step(gs, self.w, self.m, self.v, self.p16, loss_scale, hp, self.t)
        else:
            sk, self.t = Z.zero3_step(self.numel, gs, self.w_sh, self.m_sh, self.v_sh, self.p_sh,
                                      loss_scale, hp, self.t)
        return sk

    def step(self, gs):
        self.upload(gs)
        rc = A.zero_step(self.h, [g.data_ptr() for g in self.g_dev], self.loss_scale,
                         hyper(**self.hp), self.stream)
        sk = self.oracle_step(gs, self.loss_scale)
        assert (rc == A.ZERO_SKIPPED) == sk, (rc, sk)
        return sk

    def check(self, tag=""):
        wo, mo, vo, t = state_offsets(self.h, self.ws)
        assert t == self.t
        n = self.L.state_elems
        if self.view >= 0:
            ww, wm, wv = self.w, self.m, self.v
        else:
            ww, wm, wv = (np.concatenate(x) for x in (self.w_sh, self.m_sh, self.v_sh))
        compare_f32(self.ws.f32(wo, n), ww, f"master {tag}")
        compare_f32(self.ws.f32(mo, n), wm, f"m {tag}")
        compare_f32(self.ws.f32(vo, n), wv, f"v {tag}")
        if self.stage <= 2 and self.view < 0:
            for k, b in enumerate(self.bufs):
                compare_f16(b.bits(), self.reps[k], f"replica {k} {tag}")
        elif self.view >= 0:
            got = self.bufs[0].bits()
            compare_f16(got[self.b0:self.e0], self.p16, f"partition params {tag}")
            assert (got[:self.b0] == SENTINEL16).all() and (got[self.e0:] == SENTINEL16).all()
        else:
            compare_f16(self.ws.u16(self.L.off_shard16, n), np.concatenate(self.p_sh),
                        f"fp16 shards {tag}")
            for u in range(self.L.n_units):
                fb, cnt = A.zero_unit_range(self.cfg, u)
                out = GuardedF16(cnt)
                A.zero_gather_layer(self.h, u, out.ptr(), self.stream)
                want = Z.zero3_gather(self.numel, self.units, self.nd, u, self.p_sh)
                compare_f16(out.bits(), want, f"gather unit {u} {tag}")
                assert out.guards_intact()
        for b in self.bufs:
            assert b.guards_intact(), f"param buffer guard band written {tag}"
        assert self.ws.guards_intact(), f"workspace guard band written {tag}"

    def uses_tma(self):
        return A.zero_uses_tma(self.h)

    def close(self):
        A.zero_destroy(self.h)


def _run(case: Case, steps: int, inject=()):
    case.check("after init")
    skips = []
    for s in range(steps):
        gs = case.grads(s)
        for (st, k, i, bits) in inject:
            if st == s and case.b0 <= i < case.e0:
                gs[k][i - case.b0] = bits
        skips.append(case.step(gs))
        case.check(f"after step {s}")
    case.close()
    return skips


PSIS = [1, 2, 3, 7, 8, 9, 15, 16, 17, 31, 33, 40, 255, 256, 257, 1000, 4099, 8197, 70001]


@pytest.mark.parametrize("variant", VARIANTS)
@pytest.mark.parametrize("stage", [1, 2])
@pytest.mark.parametrize("nd", [1, 2, 3, 4, 5, 8, 9])
def test_stage12_grid(nd, stage, variant):
    for psi in PSIS:
        _run(Case(psi, nd, stage, variant, hp=dict(lr=1e-2, weight_decay=0.01 * (psi % 2))), 2)


@pytest.mark.parametrize("variant", VARIANTS)
@pytest.mark.parametrize("nd", [1, 2, 3, 4, 5, 8, 9])
def test_stage3_grid(nd, variant):
    rng = np.random.default_rng(nd * 10 + variant)
    for psi in PSIS:
        _run(Case(psi, nd, 3, variant, tensors=_tensor_list(rng, psi)), 2)


@pytest.mark.parametrize("variant", VARIANTS)
def test_single_rank_view_out_of_phase(variant):
    # partitions whose start is 2, 4 or 6 bytes off a 16-byte boundary in the
    # full parameter buffer, and a trailing rank that is short or empty
    for psi, nd in [(1003, 8), (8 * 1000 + 4, 8), (117, 3), (64 * 37 + 5, 64), (10, 16)]:
        for r in range(nd):
            _run(Case(psi, nd, 1 + r % 2, variant, view=r), 2)


@pytest.mark.parametrize("variant", VARIANTS)
@pytest.mark.parametrize("bits", [0x7C00, 0xFC00, 0x7E00])
def test_skip_is_global(variant, bits):
    # inf/-inf/NaN on the last rank at an element owned by rank 0, at step 1
    for stage in (1, 2, 3):
        rng = np.random.default_rng(bits + stage)
        psi, nd = 1001, 4
        tensors = _tensor_list(rng, psi) if stage == 3 else None
        skips = _run(Case(psi, nd, stage, variant, tensors=tensors), 3,
                     inject=[(1, nd - 1, 0, bits)])
        assert skips == [False, True, False]
        skips = _run(Case(psi, nd, stage, variant, tensors=tensors), 3,
                     inject=[(0, 0, psi - 1, bits), (2, 1, 500, bits)])
        assert skips == [True, False, True]


@pytest.mark.parametrize("variant", VARIANTS)
def test_skip_when_unscale_overflows(variant):
    # finite fp16 gradients, but 1/loss_scale pushes their sum past FLT_MAX
    c = Case(300, 2, 2, variant, loss_scale=1e-36, grad_dist=S.normal(1.0, 10000.0))
    skips = _run(c, 2)
    assert skips == [True, True]


def test_rank_order_of_the_sum():
    # 0.001 vanishes against 65504 in fp32; the rank order decides the result
    c = Case(16, 3, 2, A.ZERO_VARIANT_FUSED, loss_scale=1.0, hp=dict(beta1=0.0, beta2=0.0))
    c.check("init")
    g = [np.full(16, b, np.uint16) for b in
         np.array([65504.0, 0.001, -65504.0], np.float16).view(np.uint16)]
    c.step(g)
    c.check("step")
    _, mo, _, _ = state_offsets(c.h, c.ws)
    assert (c.ws.f32(mo, 16) == 0.0).all()
    c.close()


@pytest.mark.parametrize("variant", VARIANTS)
def test_zero_gradients_and_non_power_of_two_scale(variant):
    c = Case(4099, 5, 2, variant, loss_scale=3000.0, grad_dist=S.normal(0.0, 1.0))
    _run(c, 2)
    c = Case(4099, 5, 2, variant, loss_scale=3000.0, hp=dict(weight_decay=0.1, lr=0.05))
    _run(c, 3)


@pytest.mark.parametrize("variant", VARIANTS)
def test_workload_flat_1m(variant):
    wl = W.flat_1m()
    c = Case(wl.psi, wl.nd, wl.stage, variant, loss_scale=wl.loss_scale, hp=wl.hyper,
             grad_dist=wl.grad, master_dist=wl.master, seed=wl.seed)
    assert _run(c, wl.steps) == [False] * wl.steps


@pytest.mark.parametrize("variant", VARIANTS)
def test_workload_precision_stress(variant):
    wl = W.stress_16m()
    c = Case(wl.psi, wl.nd, wl.stage, variant, loss_scale=wl.loss_scale, hp=wl.hyper,
             grad_dist=wl.grad, master_dist=wl.master, seed=wl.seed)
    w_before = c.master0.copy()
    p_before = Z.f16_from_f32(w_before)
    c.check("after init")
    skips = []
    w_hist = [w_before]
    for s in range(wl.steps):
        gs = c.grads(s)
        for (st, k, i, bits) in wl.inject:
            if st == s:
                gs[k][i] = bits
        skips.append(c.step(gs))
        c.check(f"after step {s}")
        wo, _, _, _ = state_offsets(c.h, c.ws)
        w_hist.append(c.ws.f32(wo, wl.psi))
    assert skips == [False, True, False]  # the inf on rank 3 at step 2 skips it everywhere
    assert (w_hist[2].view(np.uint32) == w_hist[1].view(np.uint32)).all()
    # fp32 master absorbs every update; a direct fp16 update would lose most
    dw = (w_hist[1].astype(np.float64) - w_before).astype(np.float32)
    moved = w_hist[1] != w_before
    assert moved.mean() > 0.999
    lost = Z.direct_f16_update(p_before, dw) == p_before
    # an Adam step is ~lr = 1e-3; under RNE it is lost where half the fp16
    # spacing exceeds it, i.e. |w| >= 4 (spacing 2^-8): 2/3 of U(1, 10). The
    # pages' "2048x" rule of thumb would say |w| >= 2.048.
    big = np.abs(Z.f32_from_f16(p_before)) >= 4.0
    assert 0.6 < lost.mean() < 0.72
    assert (lost == big).mean() > 0.999
    # after the steps some fp16 params have moved although no single direct
    # fp16 update of those elements would have moved them
    p_after = c.bufs[0].bits()
    assert ((p_after != p_before) & lost).sum() > 0
    c.close()


@pytest.mark.parametrize("variant", TMA_VARIANTS)
@pytest.mark.parametrize("nd", [1, 2, 3, 4, 8, 12, 16])
def test_tma_path_runs_and_matches(nd, variant):
    # sizes with whole tiles, partial tiles, and heads/tails around them; every
    # partition in 16-byte phase, so the TMA kernels are the ones that run
    for psi in [64, 1024, 1024 * 3 + 8, 8 * 1024 * 5 + 200, 250_000, 1_000_003]:
        c = Case(psi, nd, 2, variant, hp=dict(weight_decay=0.01))
        assert c.uses_tma()
        assert _run(c, 2) == [False, False]
    c = Case(4099, 17, 2, variant)  # Nd > 16: the plain kernels
    assert not c.uses_tma()
    _run(c, 1)


@pytest.mark.parametrize("variant", TMA_VARIANTS)
@pytest.mark.parametrize("nd", [2, 4, 8, 16])
def test_tma_stage3_eligible_tensors(nd, variant):
    # tensor sizes that keep every chunk in 16-byte phase: multiples of 8 * nd
    rng = np.random.default_rng(nd)
    for trial in range(4):
        sizes = [int(x) * 8 * nd for x in rng.integers(1, 400, size=6)]
        units = [0, 0, 1, 1, 1, 2]
        c = Case(sum(sizes), nd, 3, variant, tensors=list(zip(sizes, units)))
        assert c.uses_tma()
        assert _run(c, 2, inject=[(1, nd - 1, 5, 0x7C00)]) == [False, True]


@pytest.mark.parametrize("variant", TMA_VARIANTS)
def test_tma_skip_restores_params(variant):
    c = Case(200_000, 8, 1, variant)
    assert c.uses_tma()
    assert _run(c, 3, inject=[(1, 7, 123_456, 0x7E00)]) == [False, True, False]


@pytest.mark.parametrize("variant", TMA_VARIANTS)
def test_tma_wait_that_gives_up_is_reported_and_rolled_back(variant):
    # A tile left unarmed makes the kernel's bounded waits run out (no fault):
    # the step returns ZERO_ERR_INTERNAL, nothing changes, and the next step
    # is exactly the oracle's next step. For the two-pass TMA variant the
    # unarmed tile is in the reduce pass; the update pass then does nothing.
    for psi, nd, stage in [(200_000, 8, 1), (50_000, 2, 2)]:
        c = Case(psi, nd, stage, variant)
        assert c.uses_tma()
        c.check("after init")
        c.step(c.grads(0))
        c.check("after step 0")
        A.zero_test_hold_tile(c.h, 3, 1 << 14)
        n = c.e0 - c.b0
        gs = c.grads(1)
        for k in range(c.nd):
            c.g_dev[k][:n].copy_(torch.from_numpy(gs[k].view(np.int16)))
        with pytest.raises(A.ZeroError) as ei:
            A.zero_step(c.h, [g.data_ptr() for g in c.g_dev], c.loss_scale, hyper(), c.stream)
        assert ei.value.code == A.ZERO_ERR_INTERNAL
        c.check("after the failed step: unchanged")
        assert c.step(c.grads(2)) is False
        c.check("after the next step")
        c.close()


def _async_case(stage, variant, nd=4):
    if stage == 3:
        sizes = [8 * nd * 500, 8 * nd * 37, 8 * nd * 900]
        return Case(sum(sizes), nd, 3, variant, tensors=list(zip(sizes, [0, 1, 1])),
                    grad_dist=S.normal(1e-3, 1.0), hp=dict(weight_decay=0.01))
    return Case(70_001, nd, stage, variant, grad_dist=S.normal(1e-3, 1.0),
                hp=dict(weight_decay=0.01))


@pytest.mark.parametrize("variant", VARIANTS)
@pytest.mark.parametrize("stage", [2, 3])
def test_async_steps_with_dynamic_loss_scaling(stage, variant):
    # 8 steps enqueued back to back; infs at steps 2 and 3 back the scale off
    # twice, runs of 2 good steps grow it; the oracle follows the same rule
    c = _async_case(stage, variant)
    c.check("after init")
    sc = A.zero_scaler(1024.0, 2.0, 0.5, 2)
    A.zero_async_begin(c.h, [g.data_ptr() for g in c.g_dev], sc, 0.9, 0.999, c.stream)
    scale, good, skipped = 1024.0, 0, 0
    for s in range(8):
        gs = c.grads(s)
        if s in (2, 3):
            gs[1][c.e0 - c.b0 - 1] = 0x7C00
        c.upload(gs)
        A.zero_step_async(c.h, hyper(**c.hp), c.stream)
        sk = c.oracle_step(gs, scale)
        skipped += int(sk)
        scale, good = Z.scaler_update(scale, good, sk, 2.0, 0.5, 2)
    st = A.zero_async_end(c.h, c.stream)
    assert (st.t, st.skipped, st.good_steps) == (c.t, skipped, good) == (6, 2, good)
    assert st.loss_scale == np.float32(scale)
    c.check("after the asynchronous run")
    assert c.step(c.grads(9)) is False  # the synchronous path continues from there
    c.check("after a synchronous step")
    c.close()


@pytest.mark.parametrize("variant", VARIANTS)
def test_async_step_captured_in_a_cuda_graph(variant):
    c = _async_case(2, variant, nd=8)
    cap = torch.cuda.Stream()
    sc = A.zero_scaler(4096.0, 2.0, 0.5, 3)
    with torch.cuda.stream(cap):
        A.zero_async_begin(c.h, [g.data_ptr() for g in c.g_dev], sc, 0.9, 0.999, cap.cuda_stream)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=cap):
            A.zero_step_async(c.h, hyper(**c.hp), cap.cuda_stream)
        scale, good = 4096.0, 0
        for s in range(5):
            gs = c.grads(s)
            if s == 1:
                gs[3][7] = 0x7E00
            c.upload(gs)
            graph.replay()
            sk = c.oracle_step(gs, scale)
            scale, good = Z.scaler_update(scale, good, sk, 2.0, 0.5, 3)
        st = A.zero_async_end(c.h, cap.cuda_stream)
    torch.cuda.synchronize()
    assert (st.t, st.skipped) == (c.t, 1) and st.loss_scale == np.float32(scale)
    c.check("after graph replays")
    del graph
    c.close()


def test_async_rejects_mismatched_betas_and_sync_calls():
    c = _async_case(2, A.ZERO_VARIANT_FUSED)
    A.zero_async_begin(c.h, [g.data_ptr() for g in c.g_dev], A.zero_scaler(8.0, 2.0, 0.5, 1),
                       0.9, 0.999, c.stream)
    with pytest.raises(A.ZeroError):
        A.zero_step_async(c.h, hyper(beta1=0.8), c.stream)
    with pytest.raises(A.ZeroError):
        A.zero_step(c.h, [g.data_ptr() for g in c.g_dev], 1.0, hyper(), c.stream)
    st = A.zero_async_end(c.h, c.stream)
    assert st.t == 0
    c.close()


# ---- tensors excluded from weight decay ------------------------------------
# The oracle here is the plain data-parallel step with a per-element decay
# mask on the whole vector (ZeRO leaves the math untouched); the GPU state is
# compared in its own order through the state-to-flat permutation.

def _state_perm(numel, nd, stage, psi, view):
    if stage <= 2:
        if view < 0:
            return np.arange(psi)
        b, e = Z.partition(psi, nd, view)
        return np.arange(e - b)
    offs = np.concatenate([[0], np.cumsum(numel)])
    return np.concatenate([np.arange(offs[t] + b, offs[t] + e)
                           for r in range(nd) for t, n in enumerate(numel)
                           for b, e in [Z.chunk(n, nd, r)]])


class MaskedCase(Case):
    def __init__(self, *args, **kw):
        super().__init__(*args, **kw)
        no_decay = [bool(t[2] & A.ZERO_TENSOR_NO_DECAY) if len(t) > 2 else False
                    for t in (self.tensors or [(self.psi, 0)])]
        self.mask = Z.decay_mask(self.numel, no_decay)[self.b0:self.e0].copy()
        self.perm = _state_perm(self.numel, self.nd, self.stage, self.psi, self.view)
        self.w = self.master0.copy()
        self.m = np.zeros_like(self.w)
        self.v = np.zeros_like(self.w)
        self.p16 = Z.f16_from_f32(self.w)

    def oracle_step(self, gs, loss_scale):
        sk, self.t = Z.dp_step(gs, self.w, self.m, self.v, self.p16, loss_scale,
                               Z.hyper(**self.hp), self.t, decay=self.mask)
        return sk

    def check(self, tag=""):
        wo, mo, vo, t = state_offsets(self.h, self.ws)
        assert t == self.t
        n = self.L.state_elems
        compare_f32(self.ws.f32(wo, n), self.w[self.perm], f"master {tag}")
        compare_f32(self.ws.f32(mo, n), self.m[self.perm], f"m {tag}")
        compare_f32(self.ws.f32(vo, n), self.v[self.perm], f"v {tag}")
        if self.stage <= 2 and self.view < 0:
            for k, b in enumerate(self.bufs):
                compare_f16(b.bits(), self.p16, f"replica {k} {tag}")
        elif self.view >= 0:
            compare_f16(self.bufs[0].bits()[self.b0:self.e0], self.p16, f"partition {tag}")
        else:
            compare_f16(self.ws.u16(self.L.off_shard16, n), self.p16[self.perm], f"shards {tag}")
            for u in range(self.L.n_units):
                fb, cnt = A.zero_unit_range(self.cfg, u)
                out = GuardedF16(cnt)
                A.zero_gather_layer(self.h, u, out.ptr(), self.stream)
                compare_f16(out.bits(), self.p16[fb:fb + cnt], f"gather unit {u} {tag}")
        for b in self.bufs:
            assert b.guards_intact()
        assert self.ws.guards_intact()


def _flagged(tensors, rng):
    return [(n, u, A.ZERO_TENSOR_NO_DECAY if rng.random() < 0.5 else 0) for n, u in tensors]


@pytest.mark.parametrize("variant", VARIANTS)
@pytest.mark.parametrize("stage", [1, 2, 3])
@pytest.mark.parametrize("nd", [1, 2, 3, 5, 8])
def test_no_decay_tensors_grid(nd, stage, variant):
    rng = np.random.default_rng(100 * nd + 10 * stage + variant)
    for psi in (1, 9, 257, 4099, 70001):
        tensors = _flagged(_tensor_list(rng, psi, n_max=9), rng)
        _run(MaskedCase(psi, nd, stage, variant, tensors=tensors,
                        hp=dict(lr=1e-2, weight_decay=0.1)), 2)


@pytest.mark.parametrize("variant", VARIANTS)
@pytest.mark.parametrize("view", [0, 3])
def test_no_decay_tensors_rank_view(view, variant):
    rng = np.random.default_rng(view)
    tensors = _flagged(_tensor_list(rng, 70001, n_max=12), rng)
    _run(MaskedCase(70001, 4, 1, variant, tensors=tensors, view=view,
                    hp=dict(lr=1e-2, weight_decay=0.1)), 2)


def _gpt2_like(vocab, d, layers, ctx):
    """GPT-2's tensor list at a small width, biases and layer-norm gains and
    biases excluded from weight decay (embeddings and matrices decay)."""
    ND = A.ZERO_TENSOR_NO_DECAY
    t = [(vocab * d, 0, 0), (ctx * d, 0, 0)]
    for l in range(layers):
        u = l + 1
        t += [(d, u, ND), (d, u, ND), (d * 3 * d, u, 0), (3 * d, u, ND), (d * d, u, 0), (d, u, ND),
              (d, u, ND), (d, u, ND), (d * 4 * d, u, 0), (4 * d, u, ND), (4 * d * d, u, 0), (d, u, ND)]
    t += [(d, layers + 1, ND), (d, layers + 1, ND)]
    return t


@pytest.mark.parametrize("variant", VARIANTS)
@pytest.mark.parametrize("stage", [2, 3])
def test_no_decay_gpt2_structure(stage, variant):
    tensors = _gpt2_like(1000, 96, 3, 128)
    psi = sum(n for n, _, _ in tensors)
    c = MaskedCase(psi, 8, stage, variant, tensors=tensors, loss_scale=4096.0,
                   hp=dict(lr=1e-3, weight_decay=0.01))
    if variant in TMA_VARIANTS and stage == 2:
        assert c.uses_tma()  # stage-3 shards of odd-sized tensors are out of 16-byte phase
    _run(c, 3, inject=[(1, 5, psi - 1, 0x7C00)])


@pytest.mark.parametrize("variant", VARIANTS)
def test_no_decay_async_steps(variant):
    tensors = _gpt2_like(500, 64, 2, 64)
    psi = sum(n for n, _, _ in tensors)
    c = MaskedCase(psi, 4, 2, variant, tensors=tensors, hp=dict(lr=1e-3, weight_decay=0.05))
    A.zero_async_begin(c.h, [g.data_ptr() for g in c.g_dev], A.zero_scaler(1024.0, 2.0, 0.5, 2),
                       0.9, 0.999, c.stream)
    scale, good = 1024.0, 0
    for s in range(4):
        gs = c.grads(s)
        if s == 1:
            gs[2][3] = 0x7C00
        c.upload(gs)
        A.zero_step_async(c.h, hyper(**c.hp), c.stream)
        sk = c.oracle_step(gs, scale)
        scale, good = Z.scaler_update(scale, good, sk, 2.0, 0.5, 2)
    st = A.zero_async_end(c.h, c.stream)
    assert (st.t, st.skipped) == (c.t, 1)
    c.check("after the asynchronous run")
    c.close()


@pytest.mark.parametrize("variant", [A.ZERO_VARIANT_FUSED, A.ZERO_VARIANT_TWO_PASS])
@pytest.mark.parametrize("stage", [1, 3])
def test_maximum_nd(stage, variant):
    """Nd = ZERO_MAX_ND (1024 gradient pointers and, for stage 1/2, 1024
    replica pointers in the kernels' shared-memory tables; most partitions and
    chunks a handful of elements long, the last ones empty)."""
    nd = A.ZERO_MAX_ND
    psi = 5 * nd + 37
    tensors = [(3 * nd + 5, 0), (2 * nd + 32, 1)] if stage == 3 else None
    c = Case(psi, nd, stage, variant, tensors=tensors, hp=dict(lr=1e-2, weight_decay=0.01))
    assert _run(c, 2, inject=[(1, nd - 1, 0, 0x7C00)]) == [False, True]


@pytest.mark.parametrize("variant", VARIANTS)
@pytest.mark.parametrize("hp", [dict(lr=1e-2, beta1=0.0, beta2=0.0, weight_decay=0.0),
                                dict(lr=1e-3, beta1=0.999999, beta2=0.5, weight_decay=0.0),
                                dict(lr=0.0, weight_decay=0.1),
                                dict(lr=1e-1, weight_decay=0.5, eps=1e-3)])
def test_hyperparameter_corners(variant, hp):
    """beta = 0 (bias corrections 1), beta close to 1 (tiny bias correction),
    lr = 0 (master unchanged, moments move), large decoupled weight decay."""
    _run(Case(70_001, 4, 2, variant, hp=hp), 3)
    _run(Case(8 * 4 * 999, 4, 3, variant, tensors=[(8 * 4 * 500, 0), (8 * 4 * 499, 1)], hp=hp), 2)
