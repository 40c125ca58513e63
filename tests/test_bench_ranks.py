"""The benchmark's multi-rank logic on CPU: two gloo ranks (world size 2)
take the device time of the slowest rank and report the whole job's
throughput; without a process group the same helpers are identities."""
import os
import socket

import pytest
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, times, out):
    import torch.distributed as dist
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world)
    try:
        ms = bench.max_over_ranks(times[rank], "cpu")
        value = bench.whole_job_value(1_000_000, 10, world, ms)
        out.put((rank, ms, value))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2])
def test_max_over_ranks_and_value_gloo(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    times = [100.0, 150.0]
    procs = [ctx.Process(target=_rank, args=(r, world, port, times, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(world))
    for rank, ms, value in got:
        assert ms == 150.0  # every rank sees the slowest rank's time
        assert value == pytest.approx(world * 1_000_000 * 10 / 0.150 / 1e9)


def test_single_process_identity():
    assert bench.max_over_ranks(12.5, "cpu") == 12.5
    assert bench.whole_job_value(2_000_000_000, 4, 1, 1000.0) == pytest.approx(8.0)


def test_reference_arm_other_ranks_do_nothing(monkeypatch, capsys):
    monkeypatch.setenv("RANK", "1")
    class A:  # the arguments run_reference reads
        workload, steps, warmup, gpus, variant = "flat-1m", 1, 0, 2, "fused-tma"
    bench.run_reference(A)
    assert capsys.readouterr().out == ""


def test_algorithmic_bytes_per_element():
    """The roofline's numerator: bytes per updated element of each workload,
    variant and precision, from the step's definition: (24 + 4 Nd) for stage
    1/2, (26 + 2 Nd) for stage 3, 154 per element of the Nd = 64 rank view."""
    from zero_partitioned_mixed_02_b200.synth import workloads as W
    g = W.gpt2_1p5b()
    n, floor, per, gathers = bench.algorithmic_bytes(g, "fused-tma")
    assert n == g.psi and floor == 56 * g.psi and gathers == 0
    n, floor, per, _ = bench.algorithmic_bytes(g, "two-pass-tma")
    assert floor == 56 * g.psi and sum(per.values()) == 64 * g.psi  # + 8 B of reduced gradient
    n, floor, per, _ = bench.algorithmic_bytes(g, "two-pass-tma", bf16=True)
    assert floor == 50 * g.psi and sum(per.values()) == 58 * g.psi
    ll = W.llama_2p7b()
    n, floor, _, gathers = bench.algorithmic_bytes(ll, "fused-tma")
    assert floor == 42 * ll.psi and gathers == 8 * ll.psi
    rv = W.running_example_7p5b()
    n, floor, _, _ = bench.algorithmic_bytes(rv, "fused")
    assert n == 117_187_500 and floor == 154 * n


def _agree_worker(rank, world, port, q):
    import torch
    import torch.distributed as dist
    from zero_partitioned_mixed_02_b200.distributed import agree_overflow
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    # step 7: only rank 1 overflowed (its word holds the call id); rank 0 had
    # an old overflow at step 3; nobody's kernel gave up
    words = torch.tensor([3, 0] if rank == 0 else [7, 0], dtype=torch.int32)
    agree_overflow(words)
    q.put((rank, words.tolist()))
    dist.destroy_process_group()


def test_overflow_agreement_gloo():
    """Host side of the multi-rank step: MAX of the flag words makes every
    rank see the current step's overflow (call id 7), whoever raised it."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_agree_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(60)
        assert p.exitcode == 0
    got = dict(q.get() for _ in range(2))
    assert got == {0: [7, 0], 1: [7, 0]}


@pytest.mark.parametrize("world", [1, 2, 3, 8])
def test_real_job_bytes(world):
    """The real job's per-rank byte counts: the NVLink bytes are the
    reduce-scatter and all-gather volumes of the pages' accounting for one
    rank ((Nd - 1) / Nd of 2 psi each way), and the rank's HBM bytes are the
    one-GPU step's (24 + 4 Nd) per partition element."""
    psi = 1_557_611_200
    P = -(-psi // world)
    b = bench.zero_job_bytes(psi, world, 2)
    assert b["partition"] == P
    assert b["nvlink_in"] == b["nvlink_out"] == 2 * P * (world - 1)
    assert b["hbm"] == (24 + 4 * world) * P
    b3 = bench.zero_job_bytes(psi, world, 3, n_units_elems=2 * psi)
    assert b3["nvlink_in"] == 2 * P * (world - 1) and b3["nvlink_out"] == 0
    assert b3["hbm"] == (26 + 2 * world) * P
    assert b3["nvlink_in_gathers"] == 2 * (2 * psi) * (world - 1) // world


def test_real_job_is_the_default_for_several_gpus(monkeypatch):
    """bench.py --gpus N under torchrun (WORLD_SIZE > 1) runs the real job
    unless --mode replicas asks for independent copies of the emulation."""
    calls = []
    monkeypatch.setattr(bench, "run_zero_job", lambda a: calls.append("zero"))
    monkeypatch.setattr(bench, "run_ours", lambda a: calls.append("replicas"))
    monkeypatch.setenv("WORLD_SIZE", "2")
    for argv, want in ((["bench.py", "--gpus", "2"], "zero"),
                       (["bench.py", "--gpus", "2", "--mode", "replicas"], "replicas")):
        monkeypatch.setattr("sys.argv", argv)
        bench.main()
        assert calls[-1] == want
    monkeypatch.setenv("WORLD_SIZE", "1")
    monkeypatch.setattr("sys.argv", ["bench.py"])
    bench.main()
    assert calls[-1] == "replicas"


def test_algorithmic_bytes_per_variant():
    """The floor and per-launch bytes bench.py divides by: 56 B/element for
    GPT-2's stage-2 step at Nd = 8 (fp16 with master), 50 without a master;
    the fused bfloat16 step kernel moves the floor less the replica it does
    not write, and its replica pass 4 B/element; the two passes 64."""
    wl = bench.workload("gpt2-1.5b")
    n, floor, per, gathers = bench.algorithmic_bytes(wl, "fused-tma")
    assert n == wl.psi and floor == 56 * n and per == {"step_kernel<fused>": 56 * n} and gathers == 0
    n, floor, per, _ = bench.algorithmic_bytes(wl, "fused-tma", bf16=True)
    assert floor == 50 * n and per == {"step_kernel<fused,bf16>": 48 * n, "replica_kernel": 4 * n}
    _, floor, per, _ = bench.algorithmic_bytes(wl, "two-pass-tma")
    assert floor == 56 * n and sum(per.values()) == 64 * n
    assert bench.bf16_fused_eligible(wl)
    assert not bench.bf16_fused_eligible(bench.workload("llama-2.7b"))
    assert not bench.bf16_fused_eligible(bench.workload("7.5b-rank-view"))
    ll = bench.workload("llama-2.7b")
    n, floor, _, gathers = bench.algorithmic_bytes(ll, "fused-tma")
    assert floor == 42 * n and gathers == 8 * ll.psi
