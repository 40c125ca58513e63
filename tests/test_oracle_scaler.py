"""Dynamic loss scaling rule of the oracle (a reading: the pages do not
describe loss scaling). Pinned by hand-worked sequences."""
import numpy as np

from oracle import zero_ref as Z


def run(seq, scale=1024.0, growth=2.0, backoff=0.5, interval=3):
    good = 0
    out = []
    for overflow in seq:
        scale, good = Z.scaler_update(scale, good, overflow, growth, backoff, interval)
        out.append((scale, good))
    return out


def test_backoff_and_growth_by_hand():
    # good, good, good -> x2 ; overflow -> /2 and reset ; good x3 -> x2
    got = run([False, False, False, True, False, False, False, False])
    assert got == [(1024.0, 1), (1024.0, 2), (2048.0, 0), (1024.0, 0), (1024.0, 1),
                   (1024.0, 2), (2048.0, 0), (2048.0, 1)]


def test_repeated_overflow_halves_each_time():
    got = run([True] * 5, scale=65536.0)
    assert [s for s, _ in got] == [32768.0, 16384.0, 8192.0, 4096.0, 2048.0]
    assert all(g == 0 for _, g in got)


def test_growth_never_overflows_binary32():
    big = float(np.finfo(np.float32).max) / 1.5
    got = run([False] * 3, scale=big, interval=1)
    assert all(np.isfinite(s) for s, _ in got)
    assert got[0][0] == np.float32(big)  # x2 would overflow: kept
