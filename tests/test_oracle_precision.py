"""fp16 underflow and swamping, the two failure modes the pages give for
updating fp16 weights directly ([P1] "Why you can't just delete the fp32
copies").

The page's statements are approximate; the exact rules under round to nearest
even are pinned here:
  - underflow: |x| < 2^-25 -> 0; |x| = 2^-25 -> 0 (tie to the even zero);
    2^-25 < |x| < 1.5 * 2^-24 -> 2^-24.
  - swamping: fp16(w + dw) == w iff |dw| is below half the spacing of fp16
    values next to w on dw's side (ties to even). At w = 2^e, +w/2048 is a tie
    and is lost, -w/2048 is not (the spacing below 2^e is half as large);
    |dw| <= |w|/4096 is always lost.
"""
import numpy as np

from oracle import zero_ref as Z


def h(v):
    return int(Z.f16_from_f32(np.array([v], np.float32))[0])


def hval(bits):
    return float(np.array([bits], np.uint16).view(np.float16)[0])


def test_underflow_exact_rule():
    assert h(2.0**-25) == 0
    assert h(-(2.0**-25)) == 0x8000
    assert h(np.nextafter(np.float32(2.0**-25), np.float32(1))) == 1
    assert h(1.5 * 2.0**-25) == 1
    assert h(2.0**-24) == 1
    assert h(2.0**-26) == 0
    assert hval(h(1.49 * 2.0**-24)) == 2.0**-24
    # everything strictly below 2^-25 flushes to zero
    rng = np.random.default_rng(0)
    x = (rng.random(100_000) * 2.0**-25).astype(np.float32)
    x = x[x < np.float32(2.0**-25)]
    assert (Z.f16_from_f32(x) == 0).all()


def _direct_lost(w, dw):
    w16 = Z.f16_from_f32(np.array([w], np.float32))
    out = Z.direct_f16_update(w16, np.array([dw], np.float32))
    return bool(out[0] == w16[0])


def test_swamping_exact_cases():
    for e in range(-6, 10):
        w = 2.0**e
        assert _direct_lost(w, w / 2048)          # tie, rounds back to w
        assert not _direct_lost(w, -w / 2048)     # spacing below 2^e is w/2048
        assert _direct_lost(w, w / 4096)
        assert _direct_lost(w, -w / 4096)         # tie below, rounds to even w
    assert not _direct_lost(1.999, 1.999 / 2048)  # above half a quantum


def test_swamping_always_below_quarter_quantum():
    rng = np.random.default_rng(1)
    w32 = (rng.uniform(1, 10, 50_000) * rng.choice([-1, 1], 50_000)).astype(np.float32)
    w16 = Z.f16_from_f32(w32)
    wv = Z.f32_from_f16(w16).astype(np.float64)
    frac = rng.uniform(0, 1, 50_000)
    dw = (np.abs(wv) / 4096 * frac * rng.choice([-1, 1], 50_000)).astype(np.float32)
    dw = np.where(np.abs(dw.astype(np.float64)) <= np.abs(wv) / 4096, dw, 0).astype(np.float32)
    assert (Z.direct_f16_update(w16, dw) == w16).all()


def test_swamping_threshold_2048():
    # the page's rule of thumb: updates 2048x or more smaller than the weight
    # are lost; below the exact boundary the fraction lost is total, above it
    # none are lost.
    rng = np.random.default_rng(2)
    w32 = rng.uniform(1, 2, 20_000).astype(np.float32)
    w16 = Z.f16_from_f32(w32)
    wv = Z.f32_from_f16(w16).astype(np.float64)
    big = (wv / 1000).astype(np.float32)  # well above half a quantum (1/2048 of w)
    assert (Z.direct_f16_update(w16, big) != w16).all()
    small = (wv / 5000).astype(np.float32)
    assert (Z.direct_f16_update(w16, small) == w16).all()
