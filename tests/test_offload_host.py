"""The offloaded step's host side, without a GPU.

- The host update (zero_offload_host_update: the portable build, the AVX2 +
  F16C build, and the one the step picks) against the oracle's step, bit for
  bit: with one rank and loss scale 1 the oracle's reduced gradient is the
  gradient itself, so both run the same Adam element on the same inputs.
- Its fp16 rounding over a sweep of binary32 patterns (lr = 0 leaves the
  master unchanged, so p16 = fp16(w)) against numpy's round-to-nearest-even
  conversion.
- The offload ledger: bytes crossing PCIe per step, host and device residency
  ([P2] "The Breakthrough": ZeRO-Offload moves the fp32 states and the update
  to host memory and leaves the fp16 terms on the GPU).
"""
import ctypes as C

import numpy as np
import pytest

from oracle import zero_ref as Z
from zero_partitioned_mixed_02_b200 import _abi as A


def _p(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data


def _avx2() -> bool:
    try:
        flags = open("/proc/cpuinfo").read()
    except OSError:
        return False
    return " avx2" in flags and " f16c" in flags


PATHS = [0, 1] + ([2] if _avx2() else [])


def _case(seed, n):
    rng = np.random.default_rng(seed)
    w = rng.uniform(-3, 3, n).astype(np.float32)
    w[:8] = [0.0, -0.0, 1e-40, -1e-40, 65504.0, 65519.0, 65520.0, 2.0**-25]
    m = (rng.standard_normal(n) * 1e-3).astype(np.float32)
    v = rng.uniform(0, 1e-5, n).astype(np.float32)
    g16 = (rng.standard_normal(n) * 1e-2).astype(np.float16).view(np.uint16)
    g16[8:12] = 0
    return w, m, v, g16


@pytest.mark.parametrize("path", PATHS)
@pytest.mark.parametrize("decay", [True, False])
@pytest.mark.parametrize("t", [1, 7])
def test_host_update_matches_oracle(path, decay, t):
    n = 100_003  # vector body and ragged tail
    w, m, v, g16 = _case(t * 2 + decay, n)
    hp = dict(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.05)
    # oracle: one rank, loss scale 1, step t
    ow, om, ov, op = w.copy(), m.copy(), v.copy(), np.zeros(n, np.uint16)
    sk, tt = Z.dp_step([g16], ow, om, ov, op, 1.0, Z.hyper(**hp), t - 1,
                       decay=np.full(n, 1 if decay else 0, np.uint8))
    assert not sk and tt == t
    g = Z.f32_from_f16(g16)
    hw, hm, hv, h16 = w.copy(), m.copy(), v.copy(), np.zeros(n, np.uint16)
    A.zero_offload_host_update(_p(g), _p(hw), _p(hm), _p(hv), _p(h16), n, A.zero_hyper(**hp), t, decay, path)
    for got, want in ((hw, ow), (hm, om), (hv, ov)):
        assert (got.view(np.uint32) == want.view(np.uint32)).all()
    assert (h16 == op).all()


@pytest.mark.parametrize("path", PATHS)
def test_host_fp16_rounding_sweep(path):
    # every binary32 exponent and sign, fraction bits at and around the
    # rounding boundaries of binary16 (normal and subnormal results)
    hi = np.arange(0, 1 << 16, dtype=np.uint32) << 16
    lows = np.array([0, 1, 0x0FFF, 0x1000, 0x1001, 0x1FFF, 0x2000, 0x3000, 0x7FFF, 0x8000, 0x8001,
                     0xFFFF], np.uint32)
    bits = (hi[:, None] | lows[None, :]).ravel()
    x = bits.view(np.float32)
    x = np.ascontiguousarray(x[np.isfinite(x)])
    n = x.size
    zeros = np.zeros(n, np.float32)
    w, m, v, p16 = x.copy(), zeros.copy(), zeros.copy(), np.zeros(n, np.uint16)
    A.zero_offload_host_update(_p(zeros), _p(w), _p(m), _p(v), _p(p16), n,
                               A.zero_hyper(0.0, 0.9, 0.999, 1e-8, 0.0), 1, False, path)
    assert (w.view(np.uint32) == x.view(np.uint32)).all()  # lr = 0: master unchanged
    with np.errstate(over="ignore"):
        want = x.astype(np.float16).view(np.uint16)
    assert (p16 == want).all(), int((p16 != want).sum())


def test_host_update_rejects_bad_arguments():
    a = np.zeros(4, np.float32)
    h = np.zeros(4, np.uint16)
    hp = A.zero_hyper(1e-3, 0.9, 0.999, 1e-8, 0.0)
    for t, path in ((0, 0), (1, 3), (1, -1)):
        with pytest.raises(A.ZeroError):
            A.zero_offload_host_update(_p(a), _p(a), _p(a), _p(a), _p(h), 4, hp, t, True, path)


def _numel_shard(numel, nd, r):
    return sum(e - b for b, e in (Z.chunk(n, nd, r) for n in numel))


@pytest.mark.parametrize("stage", [1, 2, 3])
def test_offload_ledger(stage):
    tensors = [(1000, 0), (17, 1), (3001, 1), (5, 2)]
    numel = [n for n, _ in tensors]
    psi, nd = sum(numel), 3
    cfg = A.Config(psi, nd, stage, tensors=tensors)
    L = A.zero_offload_bytes(cfg, 1024)
    assert L.state_elems == psi
    assert L.host_state_bytes == 12 * psi
    assert L.d2h_bytes_per_step == 4 * psi and L.h2d_bytes_per_step == 2 * psi
    assert L.chunk_elems == 1024 and L.n_chunks == (psi + 1023) // 1024
    P = max(e - b for b, e in (Z.partition(psi, nd, r) for r in range(nd)))
    Smax = max(_numel_shard(numel, nd, r) for r in range(nd))
    assert L.device_state_bytes == {1: 4 * psi, 2: 2 * psi + 2 * P, 3: 4 * Smax}[stage]
    assert L.n_out == (nd if stage <= 2 else 1)
    # slots of one fp32 and one fp16 chunk on each side
    assert L.device_bytes >= A.ZERO_OFFLOAD_SLOTS * 6 * 1024
    assert L.host_staging_bytes >= A.ZERO_OFFLOAD_SLOTS * 6 * 1024
    # the default chunk, shrunk to the state for a small problem
    assert A.zero_offload_bytes(cfg, 0).chunk_elems == (psi + 255) // 256 * 256
    mid = A.Config(1 << 24, 8, 2)
    assert A.zero_offload_bytes(mid, 0).chunk_elems == 1 << 21  # 8 chunks
    huge = A.Config(1 << 30, 8, 2)
    assert A.zero_offload_bytes(huge, 0).chunk_elems == A.ZERO_OFFLOAD_DEFAULT_CHUNK
    # rank view: one partition
    Lv = A.zero_offload_bytes(A.Config(psi, nd, 1, rank_view=2), 256)
    b, e = Z.partition(psi, nd, 2)
    assert Lv.state_elems == e - b and Lv.n_out == 1


@pytest.mark.parametrize("chunk", [100, 255, 257, -256, (1 << 30) + 256])
def test_offload_chunk_validation(chunk):
    with pytest.raises(A.ZeroError) as ei:
        A.zero_offload_bytes(A.Config(1000, 2, 2), chunk)
    assert ei.value.code == A.ZERO_ERR_ARG
