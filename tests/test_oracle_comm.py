"""Oracle communication counts pinned by simulating ring collectives.

[P1] "The part that sounds too good: communication": a ring all-reduce is a
reduce-scatter followed by an all-gather and moves 2 Psi per step; stages 1
and 2 move the same 2 Psi; stage 3 moves 3 Psi, a 1.5x increase.
[P2] "What It Enabled", stage table, communication column.

The simulation below runs the ring algorithms message by message on integer
data, checks that they compute the right thing, and counts the elements sent.
"""
import numpy as np
import pytest

from oracle import zero_ref as Z


def _chunks(psi, nd):
    return [Z.partition(psi, nd, r) for r in range(nd)]


def ring_reduce_scatter(data):
    """data[r] = rank r's full vector. Returns (owned chunks, elements sent)."""
    nd, psi = data.shape
    ch = _chunks(psi, nd)
    acc = data.copy()
    sent = 0
    # at step s, rank r sends its running partial of chunk (r - s - 1) mod nd
    # to rank r + 1, which adds its own values; after nd - 1 steps rank r holds
    # the full sum of chunk r.
    for s in range(nd - 1):
        msgs = []
        for r in range(nd):
            c = (r - s - 1) % nd
            b, e = ch[c]
            msgs.append(((r + 1) % nd, c, acc[r, b:e].copy()))
            sent += e - b
        for dst, c, payload in msgs:
            b, e = ch[c]
            acc[dst, b:e] += payload
    owned = [acc[r, ch[r][0]:ch[r][1]] for r in range(nd)]
    return owned, sent


def ring_all_gather(owned, psi):
    nd = len(owned)
    ch = _chunks(psi, nd)
    full = np.zeros((nd, psi), dtype=np.int64)
    for r in range(nd):
        full[r, ch[r][0]:ch[r][1]] = owned[r]
    sent = 0
    # at step s, rank r forwards chunk (r - s) mod nd to rank r + 1
    for s in range(nd - 1):
        msgs = []
        for r in range(nd):
            c = (r - s) % nd
            b, e = ch[c]
            msgs.append(((r + 1) % nd, b, e, full[r, b:e].copy()))
            sent += e - b
        for dst, b, e, payload in msgs:
            full[dst, b:e] = payload
    return full, sent


@pytest.mark.parametrize("nd", range(1, 10))
def test_ring_counts_brute_force(nd):
    rng = np.random.default_rng(nd)
    for psi in range(1, 41):
        data = rng.integers(-1000, 1000, size=(nd, psi)).astype(np.int64)
        owned, rs = ring_reduce_scatter(data)
        total = data.sum(axis=0)
        ch = _chunks(psi, nd)
        for r in range(nd):  # each rank owns the reduced gradients of its partition
            assert np.array_equal(owned[r], total[ch[r][0]:ch[r][1]])
        full, ag = ring_all_gather(owned, psi)
        assert all(np.array_equal(full[r], total) for r in range(nd))
        c = Z.comm_elements(psi, nd)
        assert c["reduce_scatter"] == rs, (psi, nd)
        assert c["all_gather"] == ag
        assert c["dp"] == rs + ag             # ring all-reduce = RS + AG
        assert c["stage1"] == c["dp"]         # stage 1: same volume as DP
        assert c["stage2"] == c["dp"]         # stage 2: same volume as DP
        assert c["stage3"] == rs + 2 * ag     # + the parameter gathers of fwd and bwd


def test_limits_2psi_and_3psi():
    psi = 7_500_000_000
    for nd in (64, 1024, 1 << 20):
        c = Z.comm_elements(psi, nd)
        per_rank_dp = c["dp"] / nd
        per_rank_s3 = c["stage3"] / nd
        assert per_rank_dp == pytest.approx(2 * psi * (nd - 1) / nd, rel=1e-12)
        assert per_rank_s3 == pytest.approx(3 * psi * (nd - 1) / nd, rel=1e-12)
        assert c["stage3"] / c["dp"] == pytest.approx(1.5, rel=1e-12)
    c = Z.comm_elements(psi, 1 << 20)
    assert c["dp"] / (1 << 20) / psi == pytest.approx(2.0, rel=1e-5)
    assert c["stage3"] / (1 << 20) / psi == pytest.approx(3.0, rel=1e-5)


def test_printed_communication_volumes(golden_dir):
    import os
    rows = []
    with open(os.path.join(golden_dir, "comm_pages.txt")) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                q, val, src = line.split()
                rows.append((q, float(val), src))
    assert len(rows) >= 8
    psi, nd = 10**9, 1 << 20  # the printed figures are the large-Nd limits
    c = Z.comm_elements(psi, nd)
    per_rank = {k: c[k] / nd / psi for k in ("dp", "stage1", "stage2", "stage3")}
    got = {"dp": per_rank["dp"], "s1": per_rank["stage1"], "s2": per_rank["stage2"],
           "s3": per_rank["stage3"], "s3_over_dp": c["stage3"] / c["dp"]}
    for q, val, src in rows:
        assert got[q] == pytest.approx(val, rel=1e-5), (q, val, src)
