"""Oracle binary16 conversions pinned to two independent library conversions
(numpy's and torch's) and to hand-computed values.

[P1] "Why you can't just delete the fp32 copies": the fp16 copy is derived
from the fp32 master. The pages do not name the rounding; IEEE 754 round to
nearest, ties to even, is the reading.
"""
import numpy as np
import torch

from oracle import zero_ref as Z


def _same_bits_or_both_nan_f32(a, b):
    return (a.view(np.uint32) == b.view(np.uint32)) | (np.isnan(a) & np.isnan(b))


def _same_half(a_u16, b_u16):
    a = a_u16.view(np.float16)
    b = b_u16.view(np.float16)
    return (a_u16 == b_u16) | (np.isnan(a) & np.isnan(b))


def test_half_to_float_exhaustive():
    h = np.arange(65536, dtype=np.uint16)
    ours = Z.f32_from_f16(h)
    ref = h.view(np.float16).astype(np.float32)
    assert _same_bits_or_both_nan_f32(ours, ref).all()
    ref_t = torch.from_numpy(h.view(np.int16).copy()).view(torch.float16).float().numpy()
    assert _same_bits_or_both_nan_f32(ours, ref_t).all()


def _tie_neighbourhoods():
    """Every half-quantum point of every binade the fp16 range touches, and the
    floats one ulp either side of it: all the rounding ties."""
    pts = []
    for e in range(-14, 16):  # normal binades [2^e, 2^(e+1)), quantum 2^(e-10)
        k = np.arange(2048, 4097, dtype=np.float64)
        pts.append(k * 2.0 ** (e - 11))
    pts.append(np.arange(0, 2049, dtype=np.float64) * 2.0**-25)  # subnormal half-quanta
    x = np.concatenate(pts).astype(np.float32)
    up = np.nextafter(x, np.float32(np.inf))
    dn = np.nextafter(x, np.float32(0))
    x = np.concatenate([x, up, dn])
    return np.concatenate([x, -x])


def _specials():
    vals = [0.0, -0.0, np.inf, -np.inf, np.nan, 65504.0, 65519.996, 65520.0, 65536.0,
            2.0**-24, 2.0**-25, 1.5 * 2.0**-25, 2.0**-26, 2.0**-14, 2.0**-14 - 2.0**-25,
            np.finfo(np.float32).max, np.finfo(np.float32).tiny, 1e-45, 1.0, 1.0 + 2.0**-11,
            1.0 + 3 * 2.0**-11, 2048.0, 2049.0, 2050.0, 2051.0, 4097.0, 4098.0]
    x = np.array(vals, dtype=np.float32)
    return np.concatenate([x, -x])


def test_float_to_half_ties_and_specials():
    x = np.concatenate([_tie_neighbourhoods(), _specials()])
    ours = Z.f16_from_f32(x)
    ref = x.astype(np.float16).view(np.uint16)
    assert _same_half(ours, ref).all()
    ref_t = torch.from_numpy(x).half().view(torch.int16).numpy().view(np.uint16)
    assert _same_half(ours, ref_t).all()


def test_float_to_half_strided_sweep():
    # one float in every 257 bit patterns across the whole binary32 range
    bits = np.arange(0, 2**32, 257, dtype=np.uint64).astype(np.uint32)
    x = bits.view(np.float32)
    ours = Z.f16_from_f32(x)
    ref = x.astype(np.float16).view(np.uint16)
    assert _same_half(ours, ref).all()


def test_hand_values():
    f = lambda v: int(Z.f16_from_f32(np.array([v], np.float32))[0])  # noqa: E731
    assert f(1.0) == 0x3C00
    assert f(-2.0) == 0xC000
    assert f(65504.0) == 0x7BFF
    assert f(65520.0) == 0x7C00          # halfway to 65536 rounds to even -> overflow
    assert f(65519.0) == 0x7BFF
    assert f(2.0**-24) == 0x0001         # smallest subnormal
    assert f(2.0**-14) == 0x0400         # smallest normal
    assert f(1.0 + 2.0**-11) == 0x3C00   # tie, even neighbour is 1.0
    assert f(1.0 + 3 * 2.0**-11) == 0x3C02  # tie, even neighbour is 1 + 2^-9
    assert f(-0.0) == 0x8000
    assert f(float("inf")) == 0x7C00
