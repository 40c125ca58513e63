"""The seeded generator's device path equals its host path bit for bit (fp32
values, and fp16 rounding by __float2half_rn vs numpy), for every
distribution the workloads use, at offsets that are not multiples of 8."""
import numpy as np
import pytest
import torch

from zero_partitioned_mixed_02_b200 import synth as S
from zero_partitioned_mixed_02_b200.synth import workloads as W

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a GPU", allow_module_level=True)

DISTS = [W.flat_1m().grad, W.flat_1m().master, W.stress_16m().grad, W.stress_16m().master,
         W.gpt2_1p5b().grad, S.normal(1.0, 20000.0)]


@pytest.mark.parametrize("d", range(len(DISTS)))
def test_device_equals_host(d):
    dist = DISTS[d]
    s = torch.cuda.current_stream().cuda_stream
    for index0, n in [(0, 1 << 20), (7_499_999_001, 999), (123, 4097)]:
        k = S.key(0, S.STREAM_GRAD, 2, 5)
        f = torch.empty(n, dtype=torch.float32, device="cuda")
        S.fill_f32(f.data_ptr(), n, index0, k, dist, s)
        h = torch.empty(n, dtype=torch.int16, device="cuda")
        S.fill_f16(h.data_ptr(), n, index0, k, dist, s)
        host = S.host_f32(n, index0, k, dist)
        assert (f.cpu().numpy().view(np.uint32) == host.view(np.uint32)).all()
        assert (h.cpu().numpy().view(np.uint16) == S.host_f16_bits(n, index0, k, dist)).all()
