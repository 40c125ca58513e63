"""Host side of the peer buffers of a real Nd-rank job (include/zero_peer.h,
distributed.PeerBuffers), on CPU: two gloo ranks exchange descriptors through
a fake of the library's export/open/close and must see every rank's buffers
in rank order, each opened once and closed once; the library rejects bad
arguments before any CUDA call."""
import os
import socket

import pytest
import torch.multiprocessing as mp

from zero_partitioned_mixed_02_b200 import _abi as A


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


FOREIGN = 1 << 40  # where the fake maps another process's buffer


class _FakePeers:
    log: list = []

    @staticmethod
    def export(p, n):
        return f"{os.getpid()}:{p}:{n}".encode()

    @staticmethod
    def open(d):
        pid, p, _ = d.decode().split(":")
        q = int(p) + (0 if int(pid) == os.getpid() else FOREIGN)
        _FakePeers.log.append(("open", d, q))
        return q

    @staticmethod
    def close(d, q):
        _FakePeers.log.append(("close", d, q))


def _worker(rank, world, port, nbuf, q):
    import torch.distributed as dist
    from zero_partitioned_mixed_02_b200.distributed import PeerBuffers
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        mine = [(1000 * (rank + 1) + 16 * j, 64 + j) for j in range(nbuf[rank])]
        try:
            pb = PeerBuffers(mine, api=_FakePeers)
        except ValueError as e:
            q.put((rank, "ValueError", str(e)))
            return
        ptrs = [list(r) for r in pb.ptrs]
        pb.close()
        q.put((rank, ptrs, list(_FakePeers.log)))
    finally:
        dist.destroy_process_group()


def _run(world, nbuf):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, nbuf, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = {}
    for _ in range(world):
        item = q.get(timeout=120)
        got[item[0]] = item[1:]
    for p in procs:
        p.join(60)
        assert p.exitcode == 0
    return got


@pytest.mark.parametrize("world", [2, 3])
def test_exchange_in_rank_order(world):
    got = _run(world, [2] * world)
    for rank, (ptrs, log) in got.items():
        assert len(ptrs) == world
        for k in range(world):
            expect = [1000 * (k + 1) + 16 * j + (0 if k == rank else FOREIGN) for j in range(2)]
            assert ptrs[k] == expect, (rank, k)
        opens = [(d, q) for op, d, q in log if op == "open"]
        closes = [(d, q) for op, d, q in log if op == "close"]
        assert len(opens) == 2 * world and sorted(opens) == sorted(closes)


def test_unequal_buffer_counts_fail_on_every_rank():
    got = _run(2, [2, 1])
    assert all(v[0] == "ValueError" for v in got.values())


def test_descriptor_layout():
    import ctypes as C
    assert C.sizeof(A.zero_peer_desc) == A.ZERO_PEER_DESC_BYTES == 104
    assert A.zero_peer_desc.ipc.offset == 40


def test_argument_errors_without_cuda():
    for args, code in [((0, 16), A.ZERO_ERR_ARG), ((16, 0), A.ZERO_ERR_ARG), ((8, 16), A.ZERO_ERR_ALIGN)]:
        with pytest.raises(A.ZeroError) as e:
            A.zero_peer_export(*args)
        assert e.value.code == code
    bad = bytes(104)  # magic word missing
    for f in (lambda: A.zero_peer_open(bad), lambda: A.zero_peer_close(bad, 16)):
        with pytest.raises(A.ZeroError) as e:
            f()
        assert e.value.code == A.ZERO_ERR_ARG
    with pytest.raises(A.ZeroError):
        A.zero_peer_open(bytes(10))  # wrong length
    d = A.zero_peer_desc()
    d.magic, d.bytes, d.address, d.offset = A.ZERO_PEER_MAGIC, 64, 24, 0  # misaligned address
    with pytest.raises(A.ZeroError) as e:
        A.zero_peer_open(bytes(d))
    assert e.value.code == A.ZERO_ERR_ARG
    assert A.zero_peer_open_count() == 0


class _FakeStream:
    def __init__(self):
        self.synced = 0

    def synchronize(self):
        self.synced += 1


def _barrier_worker(rank, world, port, q):
    import time

    import torch
    import torch.distributed as dist
    from zero_partitioned_mixed_02_b200.distributed import agree_overflow_any, device_barrier
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        s = _FakeStream()
        if rank == 1:
            time.sleep(1.0)  # the other rank must wait here for this one
        t0 = time.monotonic()
        device_barrier(s, None)
        waited = time.monotonic() - t0
        words = torch.tensor([0, 0] if rank == 0 else [5, 0], dtype=torch.int32)
        agree_overflow_any(words)
        q.put((rank, s.synced, waited, words.tolist()))
    finally:
        dist.destroy_process_group()


def test_device_barrier_and_agreement_gloo():
    """The gloo branch of the per-rank step's host side: device_barrier
    synchronises the stream and holds every rank until all have arrived;
    the overflow words are MAX-reduced (rank 1 overflowed on call 5)."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_barrier_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = {}
    for _ in range(2):
        rank, synced, waited, words = q.get(timeout=120)
        got[rank] = (synced, waited, words)
    for p in procs:
        p.join(60)
        assert p.exitcode == 0
    assert got[0][0] == got[1][0] == 1
    assert got[0][1] > 0.5  # rank 0 waited for the late rank
    assert got[0][2] == got[1][2] == [5, 0]
