"""Oracle ledger pinned to the values the pages print.

[P1] "Your 7.5B model's weights fit in 15 GB..." stage table and intro;
[P2] "ZeRO and the Memory Tricks", "The Mathematics" M_states(p, Nd) and the
stage table in "What It Enabled"; [P3] "DeepSpeed ZeRO: account for every
training state", "Training stores more than weights".
"""
import math
import os

import numpy as np
import pytest

from oracle import zero_ref as Z

IDX = {"dp": 0, "s1": 1, "s2": 2, "s3": 3}


def _round_sig(x: float, printed: str) -> float:
    """Round x the way the page printed `printed` (same number of significant digits)."""
    digits = len(printed.replace(".", "").lstrip("0"))
    if x == 0:
        return 0.0
    return float(f"{x:.{digits}g}")


def _golden_rows(golden_dir):
    rows = []
    with open(os.path.join(golden_dir, "ledger_pages.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            q, psi, nd, unit, val, src = line.split()
            rows.append((q, int(psi), int(nd), unit, val, src))
    return rows


def test_golden_file_present(golden_dir):
    rows = _golden_rows(golden_dir)
    assert len(rows) >= 12


def test_printed_values(golden_dir):
    for q, psi, nd, unit, printed, src in _golden_rows(golden_dir):
        div = 1e9 if unit == "GB" else float(2**30)
        if q in IDX:
            got = Z.ledger_formula(psi, nd)[IDX[q]]
        elif q == "weights16":
            got = 2.0 * psi  # the fp16 parameter term of the ledger
            assert got == Z.ledger_formula(psi, 1)[0] / 8  # 2 of the 16 bytes
        elif q == "allreduce_buf":
            # a flat fp32 buffer of the whole model: the 4-byte master term
            got = 4.0 * psi
        else:
            raise AssertionError(q)
        assert _round_sig(got / div, printed) == float(printed), (q, psi, nd, got, printed, src)


def test_worked_example_exact_bytes():
    # Psi = 7.5e9 divides evenly by 64, so the exact integer ledger equals the
    # formula to the byte: 120e9, 31.40625e9, 16.640625e9, 1.875e9.
    ex = Z.ledger_exact(7_500_000_000, 64)
    assert list(ex) == [120_000_000_000, 31_406_250_000, 16_640_625_000, 1_875_000_000]
    assert np.array_equal(ex.astype(np.float64), Z.ledger_formula(7.5e9, 64))


def test_sixteen_bytes_per_param():
    # [P1] "Where 16 bytes per parameter comes from": 2 + 2 + K with K = 12.
    for psi in (1, 7, 1000, 123456789):
        assert Z.ledger_formula(psi, 1)[0] == 16 * psi
        # with one rank every stage holds everything
        assert list(Z.ledger_formula(psi, 1)) == [16.0 * psi] * 4
        assert list(Z.ledger_exact(psi, 1)) == [16 * psi] * 4


def test_stage_limits():
    # [P1]: stage 1 is roughly a 4x cut at large Nd, stage 2 gets to 8x,
    # stage 3 scales linearly with the number of ranks.
    psi = 7.5e9
    big = 1 << 30
    f = Z.ledger_formula(psi, big)
    assert f[0] / f[1] == pytest.approx(4.0, rel=1e-6)
    assert f[0] / f[2] == pytest.approx(8.0, rel=1e-6)
    for nd in (2, 8, 64, 1024):
        a = Z.ledger_formula(psi, nd)
        b = Z.ledger_formula(psi, 2 * nd)
        assert a[3] / b[3] == pytest.approx(2.0, rel=1e-12)  # double the ranks, halve it
        assert a[0] > a[1] > a[2] > a[3]


def test_exact_matches_formula_when_divisible():
    rng = np.random.default_rng(0)
    for _ in range(200):
        nd = int(rng.integers(1, 100))
        psi = nd * int(rng.integers(1, 10**7))
        assert np.array_equal(Z.ledger_exact(psi, nd).astype(np.float64),
                              Z.ledger_formula(psi, nd))


def test_exact_is_largest_rank_under_ceil_split():
    # brute force over ranks for a non-divisible case
    psi, nd = 1003, 8
    p = math.ceil(psi / nd)
    parts = [min(p, max(0, psi - r * p)) for r in range(nd)]
    ex = Z.ledger_exact(psi, nd)
    assert ex[1] == 4 * psi + 12 * max(parts)
    assert ex[2] == 2 * psi + 14 * max(parts)
    assert ex[3] == 16 * max(parts)


def test_stage3_exact_uses_tensor_chunks():
    numel = [5, 17, 3, 1]
    nd = 4
    psi = sum(numel)
    shard = [sum(min(math.ceil(n / nd), max(0, n - r * math.ceil(n / nd))) for n in numel)
             for r in range(nd)]
    assert Z.ledger_exact(psi, nd, numel)[3] == 16 * max(shard)


def test_peak_is_not_persistent_over_nd():
    # [P3] "Check your understanding": eight-rank ZeRO-3 divides the persistent
    # lower bound by eight, but a gathered layer adds a peak that does not divide.
    numel = [4000, 96, 96, 96]  # one large layer, every tensor divisible by 8
    nd = 8
    persistent = Z.ledger_exact(sum(numel), nd, numel)[3]
    gathered_layer = 2 * max(numel)
    peak = persistent + gathered_layer
    assert persistent * nd == 16 * sum(numel)
    assert peak * nd > 16 * sum(numel)
