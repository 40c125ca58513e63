"""Randomized GPU parity across combinations the grids cover one at a time:
stage x variant x precision x Nd x ragged tensor lists with excluded tensors
x loss scale, each run for two steps against the oracle (the plain
data-parallel definition with the decay mask, or the bfloat16 step).
Deterministic (hypothesis derandomized), so a failure reproduces."""
from __future__ import annotations

import numpy as np
import pytest
import torch
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st

from zero_partitioned_mixed_02_b200 import _abi as A

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a GPU", allow_module_level=True)

from test_gpu_bf16 import Bf16Case, _run as run_bf16  # noqa: E402
from test_gpu_parity import MaskedCase, _run as run_fp16  # noqa: E402

VARIANTS = [A.ZERO_VARIANT_FUSED, A.ZERO_VARIANT_TWO_PASS, A.ZERO_VARIANT_FUSED_TMA, A.ZERO_VARIANT_TWO_PASS_TMA]


@st.composite
def jobs(draw):
    nd = draw(st.sampled_from([1, 2, 3, 4, 5, 7, 8, 9, 12, 16]))
    n_t = draw(st.integers(1, 8))
    numel = draw(st.lists(st.integers(1, 6000), min_size=n_t, max_size=n_t))
    tensors, u = [], 0
    for i, n in enumerate(numel):
        if i > 0 and draw(st.booleans()):
            u += 1
        tensors.append((n, u, draw(st.sampled_from([0, A.ZERO_TENSOR_NO_DECAY]))))
    stage = draw(st.integers(1, 3))
    bf16 = draw(st.booleans())
    # without a master the fused step exists for emulated stage 1/2 ranks, Nd >= 2
    variant = draw(st.sampled_from(VARIANTS if (not bf16 or (stage <= 2 and nd >= 2)) else VARIANTS[1::2]))
    scale = float(2 ** draw(st.integers(0, 14)))
    return nd, tensors, stage, variant, bf16, scale


@settings(max_examples=150, deadline=None, derandomize=True,
          suppress_health_check=[HealthCheck.too_slow, HealthCheck.data_too_large])
@given(jobs())
def test_random_jobs(job):
    nd, tensors, stage, variant, bf16, scale = job
    psi = sum(t[0] for t in tensors)
    hp = dict(lr=1e-2, weight_decay=0.05)
    if bf16:
        run_bf16(Bf16Case(psi, nd, stage, tensors=tensors, variant=variant, loss_scale=scale, hp=hp), 2)
    else:
        run_fp16(MaskedCase(psi, nd, stage, variant, tensors=tensors, loss_scale=scale, hp=hp), 2)
