"""Oracle partition rule checked by brute force on tiny sizes.

[P1] "The replication nobody questioned": each class of state is split across
the Nd data-parallel ranks; [P3] "What each ZeRO stage partitions". The pages
give no remainder rule; the reading is the ceil split (trailing ranks short or
empty), for the flat vector at stages 1/2 and per tensor at stage 3.
"""
import numpy as np
import pytest

from oracle import zero_ref as Z


@pytest.mark.parametrize("nd", range(1, 10))
def test_flat_partition_disjoint_covering_ordered(nd):
    for psi in range(0, 41):
        owner = np.full(psi, -1)
        prev_end = 0
        lens = []
        for r in range(nd):
            b, e = Z.partition(psi, nd, r)
            assert 0 <= b <= e <= psi
            assert b == prev_end  # ordered and contiguous
            assert (owner[b:e] == -1).all()  # disjoint
            owner[b:e] = r
            prev_end = e
            lens.append(e - b)
        assert (owner >= 0).all()  # covering
        # ceil split: lengths never increase, and every rank before the last
        # non-empty one holds exactly ceil(psi / nd) elements
        p = -(-psi // nd)
        assert lens == sorted(lens, reverse=True)
        nonempty = [r for r, x in enumerate(lens) if x > 0]
        for r in nonempty[:-1]:
            assert lens[r] == p
        if nonempty:
            assert 1 <= lens[nonempty[-1]] <= p


def test_stage3_shards_cover_every_tensor():
    rng = np.random.default_rng(1)
    for _ in range(200):
        nd = int(rng.integers(1, 10))
        numel = [int(x) for x in rng.integers(1, 30, size=rng.integers(1, 7))]
        total = 0
        for r in range(nd):
            want = 0
            for n in numel:
                b, e = Z.chunk(n, nd, r)
                want += e - b
            assert Z.shard_len(numel, nd, r) == want
            total += want
        assert total == sum(numel)


def test_running_example_partition():
    # Psi = 7.5e9, Nd = 64: 117,187,500 elements per partition
    b, e = Z.partition(7_500_000_000, 64, 0)
    assert (b, e) == (0, 117_187_500)
    b, e = Z.partition(7_500_000_000, 64, 63)
    assert e == 7_500_000_000 and e - b == 117_187_500
