"""The per-rank job of stages 1 and 2 with real peer buffers
(include/zero_peer.h, distributed.PeerRank): two processes, one rank each,
exchange CUDA IPC descriptors of their gradient and parameter buffers; rank
r's step loads partition r of both ranks' gradients through the mappings and
stores its new fp16 partition into both ranks' parameter buffers; the ranks
agree on overflow between launch and commit. Every rank's parameter buffer
and master partition must equal the plain data-parallel step of the oracle
bit for bit ([P2] "The Breakthrough": ZeRO leaves the training math
untouched), and an overflow on one rank must skip the step on both.

Both processes use the same GPU here (a node with one GPU), so the mappings
are IPC mappings of the same device rather than NVLink peers; the ranks are
ordered by stream synchronises and gloo barriers, and no kernel waits on
another process's kernel. Single-process checks of the descriptor calls come
first.
"""
from __future__ import annotations

import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from oracle import zero_ref as Z
from zero_partitioned_mixed_02_b200 import _abi as A
from zero_partitioned_mixed_02_b200 import synth as S

from gpu_common import compare_f16, compare_f32, hyper

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a GPU", allow_module_level=True)

HP = dict(lr=1e-2, weight_decay=0.05)
SCALE = 1024.0


def test_descriptor_of_this_process():
    t = torch.empty(1 << 20, dtype=torch.uint8, device="cuda")
    d0 = A.zero_peer_export(t.data_ptr(), 4096)
    d1 = A.zero_peer_export(t.data_ptr() + 4096, 8192)
    a0, a1 = A.zero_peer_desc.from_buffer_copy(d0), A.zero_peer_desc.from_buffer_copy(d1)
    assert a0.magic == A.ZERO_PEER_MAGIC and a0.bytes == 4096 and a1.bytes == 8192
    assert a1.offset - a0.offset == 4096 and a0.offset % 16 == 0
    assert a0.device == torch.cuda.current_device() and a0.process == a1.process
    # one allocation, one IPC handle
    assert bytes(a0.ipc) == bytes(a1.ipc)
    # this process's own buffer comes back unchanged and maps nothing
    assert A.zero_peer_open(d1) == t.data_ptr() + 4096
    assert A.zero_peer_open_count() == 0
    A.zero_peer_close(d1, t.data_ptr() + 4096)
    with pytest.raises(A.ZeroError) as e:
        A.zero_peer_close(d1, t.data_ptr())
    assert e.value.code == A.ZERO_ERR_ARG


def test_export_errors():
    t = torch.empty(4096, dtype=torch.uint8, device="cuda")
    with pytest.raises(A.ZeroError) as e:
        A.zero_peer_export(t.data_ptr() + 8, 16)
    assert e.value.code == A.ZERO_ERR_ALIGN
    with pytest.raises(A.ZeroError) as e:  # far past the end of the allocation
        A.zero_peer_export(t.data_ptr(), 1 << 40)
    assert e.value.code == A.ZERO_ERR_ARG
    h = torch.empty(4096, dtype=torch.uint8).pin_memory()
    with pytest.raises(A.ZeroError) as e:  # host memory
        A.zero_peer_export(h.data_ptr(), 4096)
    assert e.value.code == A.ZERO_ERR_ARG
    torch.cuda.synchronize()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _grads(psi, step, rank):
    g = S.host_f16_bits(psi, 0, S.key(4, S.STREAM_GRAD, step, rank), S.normal(1e-3, SCALE))
    return g


def _inject(g, step, rank, world):
    # step 1: an inf on the last rank, in partition 0 (owned by rank 0)
    if step == 1 and rank == world - 1:
        g[0] = 0x7C00
    return g


def _worker(rank, world, port, variants, psi, steps, q):
    from datetime import timedelta

    import torch.distributed as dist
    from zero_partitioned_mixed_02_b200.distributed import PeerRank

    torch.cuda.set_device(0)
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=timedelta(seconds=90))
    out = {}
    try:
        w0 = S.host_f32(psi, 0, S.key(4, S.STREAM_MASTER, 0, 0), S.uniform(-1.0, 1.0))
        for variant in variants:
            grad = torch.zeros(psi, dtype=torch.int16, device="cuda")
            params = torch.zeros(psi, dtype=torch.int16, device="cuda")
            P = -(-psi // world)
            b, e = min(rank * P, psi), min(rank * P + P, psi)
            job = PeerRank(grad, params, torch.from_numpy(w0[b:e].copy()).cuda(), stage=2, variant=variant)
            assert (job.begin, job.end) == (b, e)
            res = []
            for step in range(steps):
                g = _inject(_grads(psi, step, rank), step, rank, world)
                grad.copy_(torch.from_numpy(g.view(np.int16)))
                skipped = job.step(SCALE, hyper(**HP))
                wp, _, _, t = job.state()
                base = job.workspace.data_ptr()
                w = job.workspace[wp - base: wp - base + 4 * (e - b)].view(torch.float32).cpu().numpy().copy()
                res.append((skipped, t, params.cpu().numpy().view(np.uint16).copy(), w))
            mapped = A.zero_peer_open_count()
            job.close()
            out[variant] = (b, e, res, mapped, A.zero_peer_open_count())
            del job, grad, params
    except Exception as exc:  # reported to the parent, which fails the test
        out = {"error": repr(exc)}
    finally:
        dist.destroy_process_group()
        q.put((rank, out))


VARIANTS = [A.ZERO_VARIANT_FUSED, A.ZERO_VARIANT_TWO_PASS, A.ZERO_VARIANT_FUSED_TMA, A.ZERO_VARIANT_TWO_PASS_TMA]


def test_two_ranks_through_ipc_mappings():
    world, steps = 2, 3
    psi = 8000 * world - (world - 1)  # 16-byte aligned partitions, a ragged last one
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, VARIANTS, psi, steps, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = {}
    try:
        for _ in range(world):
            rank, out = q.get(timeout=300)
            got[rank] = out
    finally:
        for p in procs:
            p.join(120)
        for p in procs:  # only the processes started here, if they outlived the wait
            if p.is_alive():
                p.kill()
                p.join(30)
    assert all("error" not in out for out in got.values()), got
    assert [p.exitcode for p in procs] == [0] * world

    # the oracle: plain data-parallel mixed-precision Adam on the summed gradients
    w0 = S.host_f32(psi, 0, S.key(4, S.STREAM_MASTER, 0, 0), S.uniform(-1.0, 1.0))
    w, m, v = w0.copy(), np.zeros(psi, np.float32), np.zeros(psi, np.float32)
    p16 = Z.f16_from_f32(w)
    t = 0
    want = []
    for step in range(steps):
        gs = [_inject(_grads(psi, step, k), step, k, world) for k in range(world)]
        sk, t = Z.dp_step(gs, w, m, v, p16, SCALE, Z.hyper(**HP), t)
        want.append((sk, t, p16.copy(), w.copy()))
    assert [x[0] for x in want] == [False, True, False]

    for variant in VARIANTS:
        for rank in range(world):
            b, e, res, mapped, after = got[rank][variant]
            assert mapped in (1, 2) and after == 0, (variant, rank, mapped, after)
            for step, ((sk, tt, params, wpart), (wsk, wt, wp16, ww)) in enumerate(zip(res, want)):
                what = f"variant {variant}, rank {rank}, step {step}"
                assert sk == wsk and tt == wt, what
                compare_f16(params, wp16, f"parameters of {what}")
                compare_f32(wpart, ww[b:e], f"master of {what}")
