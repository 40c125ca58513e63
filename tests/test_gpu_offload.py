"""The offloaded step (include/zero_offload.h) against the oracle, through the
C ABI: fp32 state in host memory, Adam on the host cores, reduce and fp16
write-back on the GPU ([P2] "The Breakthrough": ZeRO-Offload changes where
the state lives, not what the step computes).

The oracle is the plain data-parallel step on the whole vector (with the
per-tensor weight-decay mask); the host state is compared in state order,
the fp16 outputs where the handle writes them. Chunks much smaller than the
state force many pipeline rounds, pieces of runs at chunk edges and reuse of
every slot.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

from oracle import zero_ref as Z
from zero_partitioned_mixed_02_b200 import _abi as A
from zero_partitioned_mixed_02_b200 import synth as S

from gpu_common import GuardedF16, compare_f16, compare_f32, hyper

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a GPU", allow_module_level=True)

ND_FLAG = A.ZERO_TENSOR_NO_DECAY


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


class OffloadCase:
    def __init__(self, psi, nd, stage, *, tensors=None, view=-1, chunk=1024, threads=3,
                 loss_scale=1024.0, hp=None, seed=0):
        self.psi, self.nd, self.stage, self.view = psi, nd, stage, view
        self.tensors = tensors or [(psi, 0)]
        self.numel = [t[0] for t in self.tensors]
        self.loss_scale = loss_scale
        self.hp = hp or dict(lr=1e-2, weight_decay=0.1)
        self.seed = seed
        self.cfg = A.Config(psi, nd, stage, rank_view=view, tensors=tensors)
        self.L = A.zero_offload_bytes(self.cfg, chunk)
        self.b0, self.e0 = Z.partition(psi, nd, view) if view >= 0 else (0, psi)
        n_own = self.e0 - self.b0
        self.master0 = S.host_f32(n_own, self.b0, S.key(seed, S.STREAM_MASTER, 0, 0), S.uniform(-1, 1))
        E = self.L.state_elems
        self.dws = torch.empty(self.L.device_bytes, dtype=torch.uint8, device="cuda")
        self.staging = torch.empty(self.L.host_staging_bytes, dtype=torch.uint8, pin_memory=True)
        self.state = np.full(3 * max(E, 1), np.nan, np.float32)
        if stage <= 2:
            self.bufs = [GuardedF16(psi) for _ in range(nd if view < 0 else 1)]
        else:
            self.bufs = [GuardedF16(E)]
        self.stream = torch.cuda.current_stream().cuda_stream
        self.h = A.zero_offload_init(self.cfg, chunk, self.dws.data_ptr(), self.L.device_bytes,
                                     self.staging.data_ptr(), self.L.host_staging_bytes,
                                     self.state.ctypes.data, self.master0.ctypes.data,
                                     [b.ptr() for b in self.bufs], threads, self.stream)
        self.g_dev = [torch.empty(max(n_own, 1), dtype=torch.int16, device="cuda") for _ in range(nd)]
        no_decay = [bool(t[2] & ND_FLAG) if len(t) > 2 else False for t in self.tensors]
        self.mask = Z.decay_mask(self.numel, no_decay)[self.b0:self.e0].copy()
        self.perm = _perm(self.numel, nd, stage, psi, view)
        self.w, self.m, self.v = self.master0.copy(), np.zeros(n_own, np.float32), np.zeros(n_own, np.float32)
        self.p16 = Z.f16_from_f32(self.w)
        self.t = 0

    def grads(self, step):
        n = self.e0 - self.b0
        return [S.host_f16_bits(n, self.b0, S.key(self.seed, S.STREAM_GRAD, step, k),
                                S.normal(1e-3, self.loss_scale)) for k in range(self.nd)]

    def step(self, gs):
        n = self.e0 - self.b0
        for k in range(self.nd):
            if n:
                self.g_dev[k][:n].copy_(torch.from_numpy(gs[k].view(np.int16)))
        rc = A.zero_offload_step(self.h, [g.data_ptr() for g in self.g_dev], self.loss_scale,
                                 hyper(**self.hp), self.stream)
        sk, self.t = Z.dp_step(gs, self.w, self.m, self.v, self.p16, self.loss_scale,
                               Z.hyper(**self.hp), self.t, decay=self.mask)
        assert (rc == A.ZERO_SKIPPED) == sk, (rc, sk)
        return sk

    def check(self, tag=""):
        torch.cuda.synchronize()
        E = self.L.state_elems
        wp, mp, vp, t = A.zero_offload_state(self.h)
        assert t == self.t
        assert wp == self.state.ctypes.data
        compare_f32(self.state[:E], self.w[self.perm], f"master {tag}")
        compare_f32(self.state[E:2 * E], self.m[self.perm], f"m {tag}")
        compare_f32(self.state[2 * E:3 * E], self.v[self.perm], f"v {tag}")
        if self.stage <= 2 and self.view < 0:
            for k, b in enumerate(self.bufs):
                compare_f16(b.bits(), self.p16, f"replica {k} {tag}")
        elif self.view >= 0:
            got = self.bufs[0].bits()
            compare_f16(got[self.b0:self.e0], self.p16, f"partition {tag}")
        else:
            compare_f16(self.bufs[0].bits(), self.p16[self.perm], f"shards {tag}")
            for u in range(A.zero_state_bytes(self.cfg).n_units):
                fb, cnt = A.zero_unit_range(self.cfg, u)
                out = GuardedF16(cnt)
                A.zero_offload_gather_layer(self.h, u, out.ptr(), self.stream)
                compare_f16(out.bits(), self.p16[fb:fb + cnt], f"gathered unit {u} {tag}")
                assert out.guards_intact()
        for b in self.bufs:
            assert b.guards_intact()

    def close(self):
        A.zero_offload_destroy(self.h)


def _run(c: OffloadCase, steps, inject=()):
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


def _tensors(rng, psi, n_max=8):
    """Random tensor list: ragged sizes, units 0, 1, ... in order, ~40 %
    excluded from weight decay."""
    k = int(rng.integers(1, min(n_max, psi) + 1))
    cuts = np.sort(rng.choice(np.arange(1, psi), size=k - 1, replace=False)) if k > 1 else []
    sizes = np.diff(np.concatenate([[0], cuts, [psi]])).astype(int)
    out, u = [], 0
    for i, n in enumerate(sizes):
        if i > 0 and rng.random() < 0.4:
            u += 1
        out.append((int(n), u, ND_FLAG if rng.random() < 0.4 else 0))
    return out


@pytest.mark.parametrize("stage", [1, 2, 3])
@pytest.mark.parametrize("nd", [1, 3, 8])
def test_offload_grid(nd, stage):
    rng = np.random.default_rng(10 * nd + stage)
    for psi, chunk in ((1, 256), (257, 256), (4099, 256), (70001, 1024), (70001, 65536)):
        tensors = _tensors(rng, psi)
        _run(OffloadCase(psi, nd, stage, tensors=tensors, chunk=chunk, threads=1 + psi % 4), 2)


@pytest.mark.parametrize("view", [0, 2, 3])
def test_offload_rank_view(view):
    rng = np.random.default_rng(view)
    _run(OffloadCase(70001, 4, 2, tensors=_tensors(rng, 70001), view=view, chunk=2048), 2)


def test_offload_skips_are_global_and_leave_state():
    psi = 50_000
    c = OffloadCase(psi, 8, 2, chunk=1024, threads=4)
    # step 1: an inf on rank 6 in a partition rank 6 does not own (rank 0's)
    skips = _run(c, 3, inject=[(1, 6, 3, 0x7C00)])
    assert skips == [False, True, False]
    c = OffloadCase(psi, 4, 3, tensors=[(20_000, 0), (30_000, 1, ND_FLAG)], chunk=512)
    assert _run(c, 2, inject=[(0, 0, psi - 1, 0x7E00)]) == [True, False]


def test_offload_matches_device_step_16m():
    """Stage 2, Nd = 8, 16,777,216 parameters, default chunk (one chunk) and a
    16-chunk pipeline: the same bits as the oracle over three steps."""
    for chunk in (0, 1 << 20):
        c = OffloadCase(1 << 24, 8, 2, chunk=chunk, threads=8, hp=dict(lr=1e-3, weight_decay=0.01))
        _run(c, 3)


def test_offload_init_validation():
    cfg = A.Config(1000, 2, 2)
    L = A.zero_offload_bytes(cfg, 256)
    dws = torch.empty(L.device_bytes, dtype=torch.uint8, device="cuda")
    pinned = torch.empty(L.host_staging_bytes, dtype=torch.uint8, pin_memory=True)
    pageable = np.empty(L.host_staging_bytes, np.uint8)
    state = np.empty(3 * 1000, np.float32)
    m0 = np.zeros(1000, np.float32)
    bufs = [torch.empty(1000, dtype=torch.int16, device="cuda") for _ in range(2)]
    s = torch.cuda.current_stream().cuda_stream
    args = dict(cfg=cfg, chunk_elems=256, device_ws=dws.data_ptr(), device_bytes=L.device_bytes,
                host_staging=pinned.data_ptr(), staging_bytes=L.host_staging_bytes,
                host_state=state.ctypes.data, master_init=m0.ctypes.data,
                param_bufs=[b.data_ptr() for b in bufs], n_threads=2, stream=s)
    for bad, code in ((dict(host_staging=pageable.ctypes.data), A.ZERO_ERR_ARG),
                      (dict(device_bytes=L.device_bytes - 1), A.ZERO_ERR_WORKSPACE),
                      (dict(n_threads=0), A.ZERO_ERR_ARG),
                      (dict(device_ws=dws.data_ptr() + 8), A.ZERO_ERR_ALIGN)):
        with pytest.raises(A.ZeroError) as ei:
            A.zero_offload_init(**{**args, **bad})
        assert ei.value.code == code
    h = A.zero_offload_init(**args)
    A.zero_offload_destroy(h)


def test_offload_checkpoint_resume():
    """Two steps, save the host state; a fresh handle restored from it and
    continued equals the original run continued, bit for bit (parameters
    rewritten from the restored master)."""
    psi, nd = 60_000, 4
    tensors = [(35_000, 0), (25_000, 1, ND_FLAG)]
    a = OffloadCase(psi, nd, 2, tensors=tensors, chunk=4096)
    for s in range(2):
        a.step(a.grads(s))
    E = a.L.state_elems
    saved = a.state[:3 * E].copy()
    for s in range(2, 4):
        a.step(a.grads(s))
    a.check("original run")
    b = OffloadCase(psi, nd, 2, tensors=tensors, chunk=4096)
    A.zero_offload_set_state(b.h, saved[:E].ctypes.data, saved[E:2 * E].ctypes.data,
                             saved[2 * E:].ctypes.data, 2, b.stream)
    torch.cuda.synchronize()
    for k, buf in enumerate(b.bufs):
        compare_f16(buf.bits(), Z.f16_from_f32(saved[:E]), f"replica {k} after restore")
    # continue b from the restored state; its oracle mirror is a's
    b.w, b.m, b.v, b.t = saved[:E].copy(), saved[E:2 * E].copy(), saved[2 * E:].copy(), 2
    b.p16 = Z.f16_from_f32(b.w)
    for s in range(2, 4):
        b.step(b.grads(s))
    b.check("resumed run")
    assert (b.state[:3 * E].view(np.uint32) == a.state[:3 * E].view(np.uint32)).all()
    a.close()
    b.close()


def test_offload_gather_rejects_stage12():
    c = OffloadCase(5000, 2, 2, chunk=1024)
    with pytest.raises(A.ZeroError) as ei:
        A.zero_offload_gather_layer(c.h, 0, GuardedF16(10).ptr(), c.stream)
    assert ei.value.code == A.ZERO_ERR_STAGE
    c.close()
