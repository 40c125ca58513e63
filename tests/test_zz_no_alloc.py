"""zero_step_static, the allocation-free step, against the existing entry point.

zero_step_static is for callers that cannot allocate device memory for a
workspace (their device memory belongs to another allocator, or they cannot
afford cudaMalloc's cost and implicit synchronisation inside a step): its
scratch lives in a fixed array inside the library. Here it is called through
the C ABI on caller-owned state and checked, on two calls in a row, against
zero_step on a handle with the two-pass variant (the same arithmetic) fed the
same gradients: master/m/v within the tests' tolerance (and bit for bit),
fp16 replicas within 1 ulp (and bit for bit), the same step count. A third
call with an inf gradient must skip on both paths. Sizes beyond the array's
limits are rejected.

This file is collected last so that a run stopping at the first failure has
already run every other test; it also passes alone in a fresh process.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

from zero_partitioned_mixed_02_b200 import _abi as A
from zero_partitioned_mixed_02_b200 import synth as S

from gpu_common import compare_f16, compare_f32, host_f32, host_u16, hyper

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a GPU", allow_module_level=True)


def _state_view(ws: torch.Tensor, ptr: int, n: int) -> torch.Tensor:
    off = ptr - ws.data_ptr()
    return ws[off: off + 4 * n].view(torch.float32)


@pytest.mark.parametrize("psi,nd", [(A.ZERO_STATIC_MAX_PSI, 4), (70001, 5), (4099, 64), (1, 1)])
def test_static_step_matches_handle_step(psi, nd):
    s = torch.cuda.current_stream().cuda_stream
    w0 = S.host_f32(psi, 0, S.key(0, S.STREAM_MASTER, 0, 0), S.uniform(-0.1, 0.1))
    gdist = S.normal(1e-3, 1024.0)
    hp = hyper(lr=1e-3, weight_decay=0.01)

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

    grads = [torch.empty(psi, dtype=torch.int16, device="cuda") for _ in range(nd)]
    gp = [g.data_ptr() for g in grads]
    for step in range(3):
        for k in range(nd):
            S.fill_f16(gp[k], psi, 0, S.key(0, S.STREAM_GRAD, step, k), gdist, s)
        if step == 2:  # an inf on the last rank: both paths must skip
            grads[nd - 1][psi // 2] = 0x7C00
        rc_h = A.zero_step(h, gp, 1024.0, hp, s)
        rc_s, t = A.zero_step_static(psi, gp, master.data_ptr(), m.data_ptr(), v.data_ptr(),
                                     [r.data_ptr() for r in reps_s], 1024.0, hp, t, s)
        want_rc = A.ZERO_SKIPPED if step == 2 else A.ZERO_OK
        assert rc_h == want_rc and rc_s == want_rc
        wp, mp, vp, th = A.zero_current_state(h)
        assert th == t == min(step + 1, 2)
        compare_f32(host_f32(master), host_f32(_state_view(ws, wp, psi)), f"master, call {step}")
        compare_f32(host_f32(m), host_f32(_state_view(ws, mp, psi)), f"m, call {step}")
        compare_f32(host_f32(v), host_f32(_state_view(ws, vp, psi)), f"v, call {step}")
        for k in range(nd):
            compare_f16(host_u16(reps_s[k]), host_u16(reps_h[k]), f"replica {k}, call {step}")
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
