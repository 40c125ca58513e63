"""The BF16 step without fp32 master weights (ZERO_PRECISION_BF16) against the
oracle's zr_bf16_step, element by element, through the C ABI ([P3] "Why
parameter count is not training memory": not every BF16 setup keeps master
weights).

The oracle runs the plain data-parallel step on the whole vector (bfloat16
gradients summed in rank order, the same skip rule, Adam on fp32 m and v,
the weight read from and rounded back to bfloat16); the GPU's m and v are
compared in state order, the bfloat16 parameters where the handle writes
them (every replica, the rank-view partition, the stage-3 shards and the
layer gathers). Gradients come from the seeded generator as binary32 and are
rounded to bfloat16 by the oracle's (pinned) conversion; both sides get the
same bits.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

from oracle import zero_ref as Z
from zero_partitioned_mixed_02_b200 import _abi as A
from zero_partitioned_mixed_02_b200 import synth as S

from gpu_common import GuardedF16, GuardedWorkspace, compare_f16, compare_f32, hyper, state_offsets

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a GPU", allow_module_level=True)

BF = A.ZERO_PRECISION_BF16
TWO = A.ZERO_VARIANT_TWO_PASS
TWO_TMA = A.ZERO_VARIANT_TWO_PASS_TMA
BF_VARIANTS = [TWO, TWO_TMA]
# the fused step without a master (emulated stage 1/2 ranks, Nd >= 2): the
# weight is read from the last replica, the new one written to the others,
# then a replica pass copies it into the last one (or, on overflow, copies
# the last one's old values back over the others)
FUSED = A.ZERO_VARIANT_FUSED
FUSED_TMA = A.ZERO_VARIANT_FUSED_TMA
BF_FUSED = [FUSED, FUSED_TMA]
NO_DECAY = A.ZERO_TENSOR_NO_DECAY


def _perm(numel, nd, stage, psi, view):
    if stage <= 2:
        if view < 0:
            return np.arange(psi)
        b, e = Z.partition(psi, nd, view)
        return np.arange(e - b)
    offs = np.concatenate([[0], np.cumsum(numel)])
    return np.concatenate([np.arange(offs[t] + b, offs[t] + e)
                           for r in range(nd) for t, n in enumerate(numel)
                           for b, e in [Z.chunk(n, nd, r)]])


class Bf16Case:
    def __init__(self, psi, nd, stage, *, tensors=None, view=-1, loss_scale=1.0, hp=None,
                 master_dist=None, grad_sigma=1e-3, seed=0, variant=TWO):
        self.psi, self.nd, self.stage, self.view = psi, nd, stage, view
        self.tensors = tensors or [(psi, 0)]
        self.numel = [t[0] for t in self.tensors]
        self.units = [t[1] for t in self.tensors]
        self.loss_scale = loss_scale
        self.hp = hp or dict(lr=1e-2, weight_decay=0.1)
        self.grad_sigma = grad_sigma
        self.seed = seed
        self.cfg = A.Config(psi, nd, stage, rank_view=view, variant=variant, tensors=tensors, precision=BF)
        self.L = A.zero_state_bytes(self.cfg)
        self.b0, self.e0 = Z.partition(psi, nd, view) if view >= 0 else (0, psi)
        n_own = self.e0 - self.b0
        self.master0 = S.host_f32(n_own, self.b0, S.key(seed, S.STREAM_MASTER, 0, 0),
                                  master_dist or S.uniform(-1.0, 1.0))
        self.ws = GuardedWorkspace(self.L.workspace_bytes)
        self.m_init = torch.from_numpy(self.master0.copy()).cuda()
        self.bufs = []
        ptrs = None
        if stage <= 2:
            self.bufs = [GuardedF16(psi) for _ in range(nd if view < 0 else 1)]
            ptrs = [b.ptr() for b in self.bufs]
        self.stream = torch.cuda.current_stream().cuda_stream
        self.h = A.zero_init(self.cfg, self.ws.ptr(), self.L.workspace_bytes, self.m_init.data_ptr(), ptrs,
                             self.stream)
        self.g_dev = [torch.empty(max(n_own, 1), dtype=torch.int16, device="cuda") for _ in range(nd)]
        no_decay = [bool(t[2] & NO_DECAY) if len(t) > 2 else False for t in self.tensors]
        self.mask = Z.decay_mask(self.numel, no_decay)[self.b0:self.e0].copy()
        self.perm = _perm(self.numel, nd, stage, psi, view)
        self.w16 = Z.bf16_from_f32(self.master0)
        self.m = np.zeros(n_own, np.float32)
        self.v = np.zeros(n_own, np.float32)
        self.t = 0

    def grads(self, step):
        n = self.e0 - self.b0
        out = []
        for k in range(self.nd):
            x = S.host_f32(n, self.b0, S.key(self.seed, S.STREAM_GRAD, step, k),
                           S.normal(self.grad_sigma, self.loss_scale))
            out.append(Z.bf16_from_f32(x))
        return out

    def upload(self, gs):
        n = self.e0 - self.b0
        for k in range(self.nd):
            if n:
                self.g_dev[k][:n].copy_(torch.from_numpy(gs[k].view(np.int16)))

    def oracle_step(self, gs, loss_scale):
        sk, self.t = Z.bf16_step(gs, self.w16, self.m, self.v, loss_scale, Z.hyper(**self.hp), self.t,
                                 decay=self.mask)
        return sk

    def step(self, gs):
        self.upload(gs)
        rc = A.zero_step(self.h, [g.data_ptr() for g in self.g_dev], self.loss_scale, hyper(**self.hp),
                         self.stream)
        sk = self.oracle_step(gs, self.loss_scale)
        assert (rc == A.ZERO_SKIPPED) == sk, (rc, sk)
        return sk

    def params(self):
        """The GPU's bfloat16 parameters of the owned range, in state order."""
        n = self.L.state_elems
        if self.stage <= 2 and self.view < 0:
            return self.bufs[0].bits()
        if self.view >= 0:
            return self.bufs[0].bits()[self.b0:self.e0]
        return self.ws.u16(self.L.off_shard16, n)

    def check(self, tag=""):
        wo, mo, vo, t = state_offsets(self.h, self.ws)
        assert t == self.t and wo is None
        n = self.L.state_elems
        compare_f32(self.ws.f32(mo, n), self.m[self.perm], f"m {tag}")
        compare_f32(self.ws.f32(vo, n), self.v[self.perm], f"v {tag}")
        if self.stage <= 2 and self.view < 0:
            for k, b in enumerate(self.bufs):
                compare_f16(b.bits(), self.w16, f"replica {k} {tag}")
        else:
            compare_f16(self.params(), self.w16[self.perm], f"parameters {tag}")
        if self.stage == 3:
            for u in range(self.L.n_units):
                fb, cnt = A.zero_unit_range(self.cfg, u)
                out = GuardedF16(cnt)
                A.zero_gather_layer(self.h, u, out.ptr(), self.stream)
                compare_f16(out.bits(), self.w16[fb:fb + cnt], f"gather unit {u} {tag}")
                assert out.guards_intact()
        for b in self.bufs:
            assert b.guards_intact()
        assert self.ws.guards_intact()

    def close(self):
        A.zero_destroy(self.h)


def _run(c, steps, inject=()):
    c.check("after init")
    skips = []
    for s in range(steps):
        gs = c.grads(s)
        for (st, k, i, bits) in inject:
            if st == s and c.b0 <= i < c.e0:
                gs[k][i - c.b0] = bits
        skips.append(c.step(gs))
        c.check(f"after step {s}")
    c.close()
    return skips


def _tensors(rng, psi, n_max=7):
    k = int(rng.integers(1, min(n_max, psi) + 1))
    cuts = np.sort(rng.choice(np.arange(1, psi), size=k - 1, replace=False)) if k > 1 else []
    sizes = np.diff(np.concatenate([[0], cuts, [psi]])).astype(int)
    out, u = [], 0
    for i, n in enumerate(sizes):
        if i > 0 and rng.random() < 0.4:
            u += 1
        out.append((int(n), u, NO_DECAY if rng.random() < 0.4 else 0))
    return out


@pytest.mark.parametrize("variant", BF_VARIANTS)
@pytest.mark.parametrize("stage", [1, 2, 3])
@pytest.mark.parametrize("nd", [1, 2, 3, 5, 8, 9])
def test_bf16_grid(nd, stage, variant):
    rng = np.random.default_rng(7 * nd + stage)
    for psi in (1, 7, 64, 257, 4099, 70001):
        _run(Bf16Case(psi, nd, stage, tensors=_tensors(rng, psi), loss_scale=float(2 ** (psi % 9)),
                      variant=variant), 2)


@pytest.mark.parametrize("variant", BF_VARIANTS)
@pytest.mark.parametrize("view", [0, 1, 3])
def test_bf16_rank_view_out_of_phase(view, variant):
    # 70001 / 4: partitions start at odd offsets, so the parameter reads are
    # out of phase with the gradient index
    rng = np.random.default_rng(view)
    _run(Bf16Case(70001, 4, 1, tensors=_tensors(rng, 70001), view=view, variant=variant), 2)


@pytest.mark.parametrize("nd", [1, 2, 4, 8])
def test_bf16_tma_passes_engage(nd):
    """Partitions in 16-byte phase: the TMA-staged passes run (whole tiles,
    partial tiles, heads and tails), with an excluded tensor."""
    for psi in (1024, 8 * 1024 * 5 + 200, 1_000_003):
        cut = psi // 3 // 64 * 64
        c = Bf16Case(psi, nd, 2, tensors=[(cut, 0), (psi - cut, 0, NO_DECAY)], variant=TWO_TMA)
        assert A.zero_uses_tma(c.h)
        _run(c, 2)


@pytest.mark.parametrize("variant", BF_VARIANTS)
def test_bf16_skips_are_global(variant):
    psi = 20_000
    assert _run(Bf16Case(psi, 8, 2, variant=variant), 3, inject=[(1, 7, 5, 0x7F80)]) == [False, True, False]
    c = Bf16Case(psi, 4, 3, tensors=[(12_000, 0), (8_000, 1, NO_DECAY)], variant=variant)
    assert _run(c, 2, inject=[(0, 0, psi - 1, 0xFFC0)]) == [True, False]


def test_bf16_subnormal_and_tiny_values():
    """Parameters and gradients near and below 2^-126 (binary32 and bfloat16
    subnormals) must not be flushed."""
    c = Bf16Case(4099, 3, 2, master_dist=S.uniform(-2.0**-120, 2.0**-120), grad_sigma=2.0**-130,
                 hp=dict(lr=2.0**-126, weight_decay=0.0))
    _run(c, 2)


@pytest.mark.parametrize("variant", BF_FUSED)
@pytest.mark.parametrize("stage", [1, 2])
@pytest.mark.parametrize("nd", [2, 3, 5, 8, 9])
def test_bf16_fused_grid(nd, stage, variant):
    rng = np.random.default_rng(11 * nd + stage)
    for psi in (1, 7, 64, 257, 4099, 70001):
        _run(Bf16Case(psi, nd, stage, tensors=_tensors(rng, psi), loss_scale=float(2 ** (psi % 9)),
                      variant=variant), 2)


@pytest.mark.parametrize("nd", [2, 4, 8, 16])
def test_bf16_fused_tma_engages(nd):
    """The TMA-staged fused kernel with the bfloat16 codec: whole tiles,
    partial tiles, heads and tails, an excluded tensor."""
    for psi in (1024, 8 * 1024 * 5 + 200, 1_000_003):
        cut = psi // 3 // 64 * 64
        c = Bf16Case(psi, nd, 2, tensors=[(cut, 0), (psi - cut, 0, NO_DECAY)], variant=FUSED_TMA)
        assert A.zero_uses_tma(c.h)
        _run(c, 2)


@pytest.mark.parametrize("variant", BF_FUSED)
def test_bf16_fused_skip_restores_every_replica(variant):
    psi = 20_000
    assert _run(Bf16Case(psi, 8, 2, variant=variant), 3, inject=[(1, 7, 5, 0x7F80)]) == [False, True, False]
    assert _run(Bf16Case(psi, 2, 1, variant=variant), 3, inject=[(0, 0, psi - 1, 0xFFC0)]) == [True, False, False]


def test_bf16_fused_wait_that_gives_up_is_rolled_back():
    """A tile left unarmed (no fault): the step returns ZERO_ERR_INTERNAL, the
    replica pass restores every replica from the last one, m/v do not switch,
    and the next step equals the oracle's next step."""
    c = Bf16Case(200_000, 8, 2, variant=FUSED_TMA)
    assert A.zero_uses_tma(c.h)
    c.check("after init")
    c.step(c.grads(0))
    c.check("after step 0")
    A.zero_test_hold_tile(c.h, 3, 1 << 14)
    c.upload(c.grads(1))
    with pytest.raises(A.ZeroError) as ei:
        A.zero_step(c.h, [g.data_ptr() for g in c.g_dev], c.loss_scale, hyper(**c.hp), c.stream)
    assert ei.value.code == A.ZERO_ERR_INTERNAL
    c.check("after the failed step: unchanged")
    c.step(c.grads(2))
    c.check("after the next step")
    c.close()


@pytest.mark.parametrize("variant", BF_VARIANTS + BF_FUSED)
def test_bf16_asynchronous_steps(variant):
    c = Bf16Case(50_000, 4, 2, tensors=[(30_000, 0), (20_000, 1, NO_DECAY)], loss_scale=1.0, variant=variant)
    c.check("after init")
    A.zero_async_begin(c.h, [g.data_ptr() for g in c.g_dev], A.zero_scaler(256.0, 2.0, 0.5, 2), 0.9, 0.999,
                       c.stream)
    scale, good, skipped = 256.0, 0, 0
    for s in range(6):
        gs = c.grads(s)
        if s == 2:
            gs[3][100] = 0x7F80
        c.upload(gs)
        A.zero_step_async(c.h, hyper(**c.hp), c.stream)
        sk = c.oracle_step(gs, scale)
        skipped += int(sk)
        scale, good = Z.scaler_update(scale, good, sk, 2.0, 0.5, 2)
    st = A.zero_async_end(c.h, c.stream)
    assert (st.t, st.skipped) == (c.t, skipped) == (5, 1)
    assert st.loss_scale == np.float32(scale)
    c.check("after the asynchronous run")
    c.close()


@pytest.mark.parametrize("variant", [TWO, FUSED_TMA])
def test_bf16_set_state(variant):
    """Resume: m, v and t restored; the parameters either stay (master NULL)
    or are rewritten from fp32 values rounded to bfloat16."""
    c = Bf16Case(10_000, 4, 2, variant=variant)
    _ = [c.step(c.grads(s)) for s in range(2)]
    n = c.L.state_elems
    rng = np.random.default_rng(1)
    m = torch.from_numpy((rng.standard_normal(n) * 1e-3).astype(np.float32)).cuda()
    v = torch.from_numpy(rng.uniform(0, 1e-6, n).astype(np.float32)).cuda()
    A.zero_set_state(c.h, 0, m.data_ptr(), v.data_ptr(), 7, c.stream)
    c.m, c.v, c.t = m.cpu().numpy(), v.cpu().numpy(), 7
    c.check("after set_state without parameters")
    w = rng.uniform(-3, 3, n).astype(np.float32)
    A.zero_set_state(c.h, torch.from_numpy(w).cuda().data_ptr(), m.data_ptr(), v.data_ptr(), 7, c.stream)
    c.w16 = Z.bf16_from_f32(w)
    c.check("after set_state with parameters")
    c.step(c.grads(5))
    c.check("after a step from the restored state")
    c.close()


@pytest.mark.parametrize("variant", [TWO_TMA, FUSED_TMA])
def test_bf16_async_step_in_a_cuda_graph(variant):
    """The bfloat16 step without master, asynchronous and captured once in a
    CUDA graph, replayed with fresh gradients (one overflowing)."""
    c = Bf16Case(40_000, 4, 2, tensors=[(24_000, 0), (16_000, 0, NO_DECAY)], variant=variant)
    c.check("after init")
    cap = torch.cuda.Stream()
    with torch.cuda.stream(cap):
        A.zero_async_begin(c.h, [g.data_ptr() for g in c.g_dev], A.zero_scaler(8.0, 2.0, 0.5, 2), 0.9, 0.999,
                           cap.cuda_stream)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=cap):
            A.zero_step_async(c.h, hyper(**c.hp), cap.cuda_stream)
        scale, good = 8.0, 0
        for s in range(5):
            gs = c.grads(s)
            if s == 2:
                gs[0][39_999] = 0x7F80
            c.upload(gs)
            graph.replay()
            sk = c.oracle_step(gs, scale)
            scale, good = Z.scaler_update(scale, good, sk, 2.0, 0.5, 2)
        st = A.zero_async_end(c.h, cap.cuda_stream)
    torch.cuda.synchronize()
    assert (st.t, st.skipped) == (c.t, 1) and st.loss_scale == np.float32(scale)
    c.check("after graph replays")
    del graph
    c.close()
