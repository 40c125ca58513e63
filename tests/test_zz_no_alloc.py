"""zero_step_static, the allocation-free step, against the existing entry point
and against the oracle.

zero_step_static is for callers that cannot allocate device memory for a
workspace (their device memory belongs to another allocator, or they cannot
afford cudaMalloc's cost and implicit synchronisation inside a step): its
scratch lives in a fixed array inside the library. Here it is called through
the C ABI on caller-owned state and checked, call after call, against
zero_step on a handle with the two-pass variant (the same arithmetic) fed the
same gradients, and against the oracle's data-parallel step (the definition
of the result): master/m/v within the tests' tolerance (and bit for bit),
fp16 replicas within 1 ulp (and bit for bit), the same step count. Four calls:
two ordinary ones, one with an inf gradient that must skip on every path, and
an ordinary one after the skip (the overflow word is cleared between calls).
The sizes include ones where some ranks own empty partitions. Sizes beyond the
array's limits are rejected.

This file is collected last so that a run stopping at the first failure has
already run every other test; it also passes alone in a fresh process.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

from oracle import zero_ref as Z
from zero_partitioned_mixed_02_b200 import _abi as A
from zero_partitioned_mixed_02_b200 import synth as S

from gpu_common import compare_f16, compare_f32, dev_u16, host_f32, host_u16, hyper

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a GPU", allow_module_level=True)

HP = dict(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.01)
SCALE = 1024.0


def _state_view(ws: torch.Tensor, ptr: int, n: int) -> torch.Tensor:
    off = ptr - ws.data_ptr()
    return ws[off: off + 4 * n].view(torch.float32)


@pytest.mark.parametrize("psi,nd", [(A.ZERO_STATIC_MAX_PSI, 4), (70001, 5), (4099, 64), (1, 1),
                                    (3, 8), (17, 64)])
def test_static_step_matches_handle_step_and_oracle(psi, nd):
    s = torch.cuda.current_stream().cuda_stream
    w0 = S.host_f32(psi, 0, S.key(0, S.STREAM_MASTER, 0, 0), S.uniform(-0.1, 0.1))
    gdist = S.normal(1e-3, SCALE)
    hp = hyper(**HP)

    # the existing entry point: a handle with its workspace
    cfg = A.Config(psi, nd, 2, variant=A.ZERO_VARIANT_TWO_PASS)
    L = A.zero_state_bytes(cfg)
    ws = torch.empty(L.workspace_bytes, dtype=torch.uint8, device="cuda")
    m_init = torch.from_numpy(w0.copy()).cuda()
    reps_h = [torch.zeros(psi, dtype=torch.int16, device="cuda") for _ in range(nd)]
    h = A.zero_init(cfg, ws.data_ptr(), L.workspace_bytes, m_init.data_ptr(),
                    [r.data_ptr() for r in reps_h], s)

    # the allocation-free entry point: state owned by the caller
    master = torch.from_numpy(w0.copy()).cuda()
    m = torch.zeros(psi, dtype=torch.float32, device="cuda")
    v = torch.zeros(psi, dtype=torch.float32, device="cuda")
    reps_s = [torch.zeros(psi, dtype=torch.int16, device="cuda") for _ in range(nd)]
    t = 0

    # the oracle: the plain data-parallel step on the CPU
    ow, om, ov = w0.copy(), np.zeros(psi, np.float32), np.zeros(psi, np.float32)
    op16 = Z.f16_from_f32(w0)
    ot = 0
    ohp = Z.hyper(**HP)

    for step in range(4):
        gs = [S.host_f16_bits(psi, 0, S.key(0, S.STREAM_GRAD, step, k), gdist) for k in range(nd)]
        if step == 2:  # an inf on the last rank: every path must skip
            gs[nd - 1][psi // 2] = 0x7C00
        grads = [dev_u16(g) for g in gs]
        gp = [g.data_ptr() for g in grads]
        rc_h = A.zero_step(h, gp, SCALE, hp, s)
        rc_s, t = A.zero_step_static(psi, gp, master.data_ptr(), m.data_ptr(), v.data_ptr(),
                                     [r.data_ptr() for r in reps_s], SCALE, hp, t, s)
        skipped, ot = Z.dp_step(gs, ow, om, ov, op16, SCALE, ohp, ot)
        want_rc = A.ZERO_SKIPPED if step == 2 else A.ZERO_OK
        assert rc_h == want_rc and rc_s == want_rc and skipped == (step == 2)
        wp, mp, vp, th = A.zero_current_state(h)
        assert th == t == ot == (step + 1 if step < 2 else step)
        got = {"master": host_f32(master), "m": host_f32(m), "v": host_f32(v)}
        handle = {"master": host_f32(_state_view(ws, wp, psi)), "m": host_f32(_state_view(ws, mp, psi)),
                  "v": host_f32(_state_view(ws, vp, psi))}
        oracle = {"master": ow, "m": om, "v": ov}
        for name in got:
            compare_f32(got[name], oracle[name], f"{name} vs oracle, call {step}")
            compare_f32(got[name], handle[name], f"{name} vs zero_step, call {step}")
        for k in range(nd):
            compare_f16(host_u16(reps_s[k]), op16, f"replica {k} vs oracle, call {step}")
            compare_f16(host_u16(reps_s[k]), host_u16(reps_h[k]), f"replica {k} vs zero_step, call {step}")
    A.zero_destroy(h)


def test_static_step_rejects_sizes_beyond_its_array():
    s = torch.cuda.current_stream().cuda_stream
    buf = torch.zeros(64, dtype=torch.float32, device="cuda")
    p = buf.data_ptr()
    hp = hyper()
    with pytest.raises(A.ZeroError) as ei:
        A.zero_step_static(A.ZERO_STATIC_MAX_PSI + 1, [p], p, p, p, [p], 1.0, hp, 0, s)
    assert ei.value.code == A.ZERO_ERR_ARG
    with pytest.raises(A.ZeroError) as ei:
        A.zero_step_static(16, [p] * (A.ZERO_STATIC_MAX_ND + 1), p, p, p,
                           [p] * (A.ZERO_STATIC_MAX_ND + 1), 1.0, hp, 0, s)
    assert ei.value.code == A.ZERO_ERR_ARG
    with pytest.raises(A.ZeroError) as ei:
        A.zero_step_static(16, [p + 4], p, p, p, [p], 1.0, hp, 0, s)
    assert ei.value.code == A.ZERO_ERR_ALIGN
