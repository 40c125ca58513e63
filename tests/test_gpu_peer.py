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


CASES = {
    # stage 2, fp16 gradients and parameters with fp32 master, every variant
    "fp16": dict(stage=2, precision=A.ZERO_PRECISION_FP16, tensors=None, inf=0x7C00,
                 variants=[A.ZERO_VARIANT_FUSED, A.ZERO_VARIANT_TWO_PASS, A.ZERO_VARIANT_FUSED_TMA,
                           A.ZERO_VARIANT_TWO_PASS_TMA]),
    # stage 1, bfloat16 without master, a tensor excluded from weight decay
    "bf16": dict(stage=1, precision=A.ZERO_PRECISION_BF16, inf=0x7F80,
                 tensors=[(5000, 0), (10999, 0, A.ZERO_TENSOR_NO_DECAY)],
                 variants=[A.ZERO_VARIANT_TWO_PASS, A.ZERO_VARIANT_TWO_PASS_TMA]),
}


def _scale(case):
    return 1.0 if case["precision"] == A.ZERO_PRECISION_BF16 else SCALE


def _grads(case, psi, step, rank, world):
    key = S.key(4, S.STREAM_GRAD, step, rank)
    if case["precision"] == A.ZERO_PRECISION_BF16:
        g = Z.bf16_from_f32(S.host_f32(psi, 0, key, S.normal(1e-3, 1.0)))
    else:
        g = S.host_f16_bits(psi, 0, key, S.normal(1e-3, SCALE))
    # step 1: an inf on the last rank, in partition 0 (owned by rank 0)
    if step == 1 and rank == world - 1:
        g[0] = case["inf"]
    return g


def _worker(rank, world, port, name, psi, steps, q):
    from datetime import timedelta

    import torch.distributed as dist
    from zero_partitioned_mixed_02_b200.distributed import PeerRank

    case = CASES[name]
    bf16 = case["precision"] == A.ZERO_PRECISION_BF16
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=timedelta(seconds=90))
    out = {}
    try:
        w0 = S.host_f32(psi, 0, S.key(4, S.STREAM_MASTER, 0, 0), S.uniform(-1.0, 1.0))
        for variant in case["variants"]:
            grad = torch.zeros(psi, dtype=torch.int16, device="cuda")
            params = torch.zeros(psi, dtype=torch.int16, device="cuda")
            P = -(-psi // world)
            b, e = min(rank * P, psi), min(rank * P + P, psi)
            job = PeerRank(grad, params, torch.from_numpy(w0[b:e].copy()).cuda(), stage=case["stage"],
                           variant=variant, precision=case["precision"], tensors=case["tensors"])
            assert (job.begin, job.end) == (b, e)
            res = []
            for step in range(steps):
                grad.copy_(torch.from_numpy(_grads(case, psi, step, rank, world).view(np.int16)))
                skipped = job.step(_scale(case), hyper(**HP))
                wp, mp, _, t = job.state()
                src = mp if bf16 else wp  # no master in bfloat16: check the first moment
                base = job.workspace.data_ptr()
                x = job.workspace[src - base: src - base + 4 * (e - b)].view(torch.float32).cpu().numpy().copy()
                res.append((skipped, t, params.cpu().numpy().view(np.uint16).copy(), x))
            mapped = A.zero_peer_open_count()
            job.close()
            out[variant] = (b, e, res, mapped, A.zero_peer_open_count())
            del job, grad, params
    except Exception as exc:  # reported to the parent, which fails the test
        out = {"error": repr(exc)}
    finally:
        dist.destroy_process_group()
        q.put((rank, out))


@pytest.mark.parametrize("name", list(CASES))
def test_two_ranks_through_ipc_mappings(name):
    case = CASES[name]
    world, steps = 2, 3
    psi = 8000 * world - (world - 1)  # 16-byte aligned partitions, a ragged last one
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, name, psi, steps, q)) for r in range(world)]
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
    bf16 = case["precision"] == A.ZERO_PRECISION_BF16
    tensors = case["tensors"]
    mask = Z.decay_mask([x[0] for x in tensors], [len(x) > 2 for x in tensors]) if tensors else None
    w0 = S.host_f32(psi, 0, S.key(4, S.STREAM_MASTER, 0, 0), S.uniform(-1.0, 1.0))
    w, m, v = w0.copy(), np.zeros(psi, np.float32), np.zeros(psi, np.float32)
    p16 = Z.bf16_from_f32(w) if bf16 else Z.f16_from_f32(w)
    t = 0
    want = []
    for step in range(steps):
        gs = [_grads(case, psi, step, k, world) for k in range(world)]
        if bf16:
            sk, t = Z.bf16_step(gs, p16, m, v, _scale(case), Z.hyper(**HP), t, decay=mask)
        else:
            sk, t = Z.dp_step(gs, w, m, v, p16, _scale(case), Z.hyper(**HP), t, decay=mask)
        want.append((sk, t, p16.copy(), (m if bf16 else w).copy()))
    assert [x[0] for x in want] == [False, True, False]

    for variant in case["variants"]:
        for rank in range(world):
            b, e, res, mapped, after = got[rank][variant]
            assert mapped in (1, 2) and after == 0, (variant, rank, mapped, after)
            for step, ((sk, tt, params, x), (wsk, wt, wp16, wx)) in enumerate(zip(res, want)):
                what = f"{name}, variant {variant}, rank {rank}, step {step}"
                assert sk == wsk and tt == wt, what
                compare_f16(params, wp16, f"parameters of {what}")
                compare_f32(x, wx[b:e], f"{'m' if bf16 else 'master'} of {what}")


# stage 3: each rank keeps its shard in its workspace; after every step each
# rank gathers every layer unit from both ranks' shards through the mappings
TENSORS3 = [(8192, 0), (4096, 0), (40001, 1), (2048, 1), (777, 2), (5000, 3)]


def _shards(x, numel, nd, r):
    out, off = [], 0
    for n in numel:
        b, e = Z.chunk(n, nd, r)
        out.append(x[off + b: off + e])
        off += n
    return np.concatenate(out)


def _worker3(rank, world, port, variants, steps, q):
    from datetime import timedelta

    import torch.distributed as dist
    from zero_partitioned_mixed_02_b200.distributed import PeerRank

    torch.cuda.set_device(0)
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=timedelta(seconds=90))
    out = {}
    try:
        psi = sum(t[0] for t in TENSORS3)
        n_units = TENSORS3[-1][1] + 1
        w0 = S.host_f32(psi, 0, S.key(6, S.STREAM_MASTER, 0, 0), S.uniform(-1.0, 1.0))
        for variant in variants:
            grad = torch.zeros(psi, dtype=torch.int16, device="cuda")
            job = PeerRank(grad, None, torch.from_numpy(w0.copy()).cuda(), stage=3, variant=variant,
                           tensors=TENSORS3)
            n = A.zero_state_bytes(job.cfg).state_elems
            res = []
            for step in range(steps):
                g = S.host_f16_bits(psi, 0, S.key(6, S.STREAM_GRAD, step, rank), S.normal(1e-3, SCALE))
                if step == 1 and rank == 0:
                    g[psi - 1] = 0xFC00  # -inf on rank 0, in the last tensor's last chunk (rank 1's)
                grad.copy_(torch.from_numpy(g.view(np.int16)))
                skipped = job.step(SCALE, hyper(**HP))
                wp, _, _, t = job.state()
                base = job.workspace.data_ptr()
                w = job.workspace[wp - base: wp - base + 4 * n].view(torch.float32).cpu().numpy().copy()
                units = []
                for u in range(n_units):
                    buf = torch.empty(job.unit_range(u)[1], dtype=torch.int16, device="cuda")
                    job.gather(u, buf)
                    units.append(buf.cpu().numpy().view(np.uint16).copy())
                res.append((skipped, t, w, units))
            mapped = A.zero_peer_open_count()
            job.close()
            out[variant] = (res, mapped, A.zero_peer_open_count())
            del job, grad
    except Exception as exc:  # reported to the parent, which fails the test
        out = {"error": repr(exc)}
    finally:
        dist.destroy_process_group()
        q.put((rank, out))


def test_stage3_ranks_through_ipc_mappings():
    world, steps = 2, 3
    variants = CASES["fp16"]["variants"]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker3, args=(r, world, port, variants, steps, q)) for r in range(world)]
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

    numel = [t[0] for t in TENSORS3]
    unit_of = [t[1] for t in TENSORS3]
    psi = sum(numel)
    w0 = S.host_f32(psi, 0, S.key(6, S.STREAM_MASTER, 0, 0), S.uniform(-1.0, 1.0))
    w_sh = [_shards(w0, numel, world, r).copy() for r in range(world)]
    m_sh = [np.zeros_like(x) for x in w_sh]
    v_sh = [np.zeros_like(x) for x in w_sh]
    p_sh = [Z.f16_from_f32(x) for x in w_sh]
    t = 0
    want = []
    for step in range(steps):
        gs = [S.host_f16_bits(psi, 0, S.key(6, S.STREAM_GRAD, step, k), S.normal(1e-3, SCALE))
              for k in range(world)]
        if step == 1:
            gs[0][psi - 1] = 0xFC00
        sk, t = Z.zero3_step(numel, gs, w_sh, m_sh, v_sh, p_sh, SCALE, Z.hyper(**HP), t)
        units = [Z.zero3_gather(numel, unit_of, world, u, p_sh) for u in range(unit_of[-1] + 1)]
        want.append((sk, t, [x.copy() for x in w_sh], units))
    assert [x[0] for x in want] == [False, True, False]

    for variant in variants:
        for rank in range(world):
            res, mapped, after = got[rank][variant]
            assert mapped in (1, 2) and after == 0, (variant, rank, mapped, after)
            for step, ((sk, tt, w, units), (wsk, wt, ww, wunits)) in enumerate(zip(res, want)):
                what = f"stage 3, variant {variant}, rank {rank}, step {step}"
                assert sk == wsk and tt == wt, what
                compare_f32(w, ww[rank], f"master shard of {what}")
                for u, (x, y) in enumerate(zip(units, wunits)):
                    compare_f16(x, y, f"unit {u} of {what}")


@pytest.mark.parametrize("workload", ["stress-16m", "llama-block"])
def test_bench_real_job_two_ranks(workload):
    """bench.py's real-job mode (the default for --gpus N > 1), launched like
    the multi-GPU benchmark (torchrun, one process per rank), here with two
    ranks on this one GPU over gloo: peer mappings of the same device instead
    of NVLink peers, no NCCL comparison. It must exit 0 and print one line
    describing the Nd = 2 job (stage 2, and stage 3 with the rank gathers)."""
    import json
    import os
    import subprocess
    import sys

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    cmd = ["timeout", "-k", "60", "600", sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
           "--nproc-per-node", "2", "--master-addr", "127.0.0.1", "--master-port", str(_free_port()),
           os.path.join(root, "bench.py"), "--gpus", "2", "--backend", "gloo", "--workload", workload,
           "--steps", "3", "--warmup", "3", "--e2e-steps", "2"]
    out = subprocess.run(cmd, capture_output=True, text=True, cwd=root)
    assert out.returncode == 0, out.stdout[-2000:] + out.stderr[-4000:]
    lines = [x for x in out.stdout.splitlines() if x.startswith("{")]
    assert len(lines) == 1, out.stdout[-2000:]
    line = json.loads(lines[0])
    assert line["n_gpus"] == 2 and line["config"]["nd"] == 2 and line["scaling"] == "strong"
    assert line["steps"] == 3 and line["value"] > 0 and line["gpu_launches"] > 0
    assert line["roofline"]["bound"] == "nvlink" and line["roofline"]["kernel_ms"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 2 * line["config"]["psi"]
    assert "nccl_rs_ag" not in line  # gloo: no NCCL leg
    if workload == "llama-block":
        assert line["config"]["stage"] == 3 and line["gathers"]["launches_per_step"] == 6
