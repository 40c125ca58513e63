#!/usr/bin/env python
"""Benchmark of the ZeRO partitioned mixed-precision Adam step on B200.

One step = one pass of the hot path over one batch of synthetic gradients:
the emulated reduce-scatter of Nd fp16 gradient vectors (rank-ordered fp32
sum), unscale + global overflow check, Adam on the fp32 master/m/v of every
partition, fp16 cast and all-gather write-back (stage 1/2) or shard write
plus the forward and backward layer gathers (stage 3). Inputs are resident in
HBM when the timed region starts; everything moved per step (tens of GB at
the default workload) exceeds the 126 MB L2, so no flush is needed.

Prints ONE JSON line (rank 0). ``--impl reference`` times the plain CPU
oracle on a bounded sample of the same workload instead.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--variant fused-tma|fused|two-pass] [--impl ours|reference]
"""
from __future__ import annotations

import argparse
import csv
import hashlib
import io
import json
import os
import re
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "ZeRO Adam step Gparams/s and HBM GB/s (% of peak) on 1 B200 vs CPU oracle"
UNIT = "Gparams/s"
FALLBACK_HBM_GBS = 6650.0
CSRC = os.path.join(ROOT, "zero_partitioned_mixed_02_b200", "csrc")

WORKLOADS = {
    "flat-1m": 1, "stress-16m": 2, "gpt2-1.5b": 3, "7.5b-rank-view": 4, "llama-2.7b": 5,
}
PROFILE_WORKLOADS = ("flat-64m", "llama-block", "view-1g")


def parse_args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=60)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--mode", choices=["zero", "replicas"], default=None,
                   help="with --gpus N > 1: 'zero' (default) runs the real job, Nd = N ranks, one "
                        "partition per GPU over peer memory; 'replicas' runs N independent copies of the "
                        "one-GPU emulation")
    p.add_argument("--backend", choices=["nccl", "gloo"], default="nccl",
                   help="process-group backend of the real job (gloo: ranks may share one GPU; "
                        "no NCCL comparison)")
    p.add_argument("--workload", choices=sorted(WORKLOADS) + sorted(PROFILE_WORKLOADS), default="gpt2-1.5b",
                   help="the five configurations, or a small profiling case of their kernels "
                        "(flat-64m: the stage-2 step at psi = 2^26; llama-block: one Llama block, stage 3; "
                        "view-1g: the rank view at psi = 2^30, Nd = 64)")
    p.add_argument("--variant", choices=["fused-tma", "fused", "two-pass", "two-pass-tma"], default="fused-tma")
    p.add_argument("--precision", choices=["fp16", "bf16"], default="fp16",
                   help="bf16: bfloat16 gradients and parameters without fp32 master weights (the fused "
                        "variants need a second replica to roll back to: stage 1/2 with Nd >= 2; otherwise a "
                        "fused --variant becomes two-pass-tma)")
    p.add_argument("--async", dest="async_steps", action="store_true",
                   help="time zero_step_async: steps enqueued back to back, no host sync")
    p.add_argument("--prefetch", action="store_true",
                   help="stage 3: also time the layer gathers against a stand-in GEMM, "
                        "one after the other vs prefetched on a side stream")
    p.add_argument("--offload", action="store_true",
                   help="time the offloaded step (fp32 state and Adam on the host) instead")
    p.add_argument("--offload-threads", type=int, default=0,
                   help="host threads of the offloaded update (0: every core this process may use)")
    p.add_argument("--offload-chunk", type=int, default=0,
                   help="elements per pipeline chunk of the offloaded step (0: the library default)")
    p.add_argument("--e2e-steps", type=int, default=6)
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-per-config", action="store_true",
                   help="time only --workload (by default a one-GPU fp16 synchronous run of a workload "
                        "with psi >= 1B also times the other two under per_config)")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--cpu-seconds", type=float, default=10.0,
                   help="target CPU time of the oracle baseline sample")
    return p.parse_args()


def bf16_fused_eligible(wl) -> bool:
    """The fused step without an fp32 master needs a second copy of the weights
    to roll back to: emulated stage 1/2 ranks with Nd >= 2."""
    return wl.stage <= 2 and wl.rank_view < 0 and wl.nd >= 2


def workload(name):
    from zero_partitioned_mixed_02_b200.synth import workloads as W
    if name in W.PROFILE:
        return W.PROFILE[name]()
    return W.ALL[WORKLOADS[name]]()


# ---------------------------------------------------------------- bytes
def owned_range(wl):
    if wl.rank_view >= 0:
        p = -(-wl.psi // wl.nd)
        b = min(wl.rank_view * p, wl.psi)
        return b, min(b + p, wl.psi)
    return 0, wl.psi


def algorithmic_bytes(wl, variant, bf16=False):
    """Minimum bytes one step of the method must move (the floor), and per
    launch of the dominant kernel. n = elements this GPU updates."""
    b0, e0 = owned_range(wl)
    n = e0 - b0
    grads = 2 * wl.nd * n                    # every rank's 16-bit gradient of each element
    n_out = wl.nd if (wl.stage <= 2 and wl.rank_view < 0) else 1
    if bf16:
        state = 16 * n + 2 * n               # fp32 m, v read and written; the bf16 weight read
    else:
        state = 24 * n                       # fp32 master, m, v read and written
    params = 2 * n * n_out                   # 16-bit write-back to every replica / the shard
    floor = grads + state + params
    if variant in ("fused", "fused-tma") and bf16:
        # without a master: the step reads the weight from the last replica and
        # writes the others; the replica pass then copies one replica (2 + 2 B)
        per_launch = {"step_kernel<fused,bf16>": floor - 2 * n, "replica_kernel": 4 * n}
    elif variant in ("fused", "fused-tma"):
        per_launch = {"step_kernel<fused>": floor}
    else:
        per_launch = {"step_kernel<reduce>": grads + 4 * n,
                      "step_kernel<update>": 4 * n + state + params}
    gathers = 8 * wl.psi if wl.stage == 3 else 0  # 2 psi read + 2 psi written, forward and back
    return n, floor, per_launch, gathers


# ---------------------------------------------------------------- environment
def stream_copy_gbs(n_bytes=1 << 32, reps=10):
    """This library's own copy kernel (zero_stream_copy) on n_bytes, read +
    written bytes per second, median of reps: a same-run reference beside the
    pool's measured peak."""
    import torch

    from zero_partitioned_mixed_02_b200 import _abi as A

    src = torch.empty(n_bytes, dtype=torch.uint8, device="cuda")
    dst = torch.empty_like(src)
    s = torch.cuda.current_stream()
    A.zero_stream_copy(dst.data_ptr(), src.data_ptr(), n_bytes, s.cuda_stream)
    ms = []
    for _ in range(reps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(s)
        A.zero_stream_copy(dst.data_ptr(), src.data_ptr(), n_bytes, s.cuda_stream)
        b.record(s)
        b.synchronize()
        ms.append(a.elapsed_time(b))
    del src, dst
    torch.cuda.empty_cache()
    return 2 * n_bytes / (sorted(ms)[len(ms) // 2] / 1e3) / 1e9


def measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


# device sources each variant's step kernel is built from
KERNEL_FILES = {
    "fused-tma": ("zero_device.cuh", "zero_internal.h", "zero_tma.cuh", "zero_tma.cu"),
    "fused": ("zero_device.cuh", "zero_internal.h", "zero_kernels.cu"),
    "two-pass": ("zero_device.cuh", "zero_internal.h", "zero_kernels.cu"),
    "two-pass-bf16": ("zero_device.cuh", "zero_internal.h", "zero_kernels.cu"),
    "two-pass-tma": ("zero_device.cuh", "zero_internal.h", "zero_tma.cuh", "zero_tma_pass.cu"),
    "two-pass-tma-bf16": ("zero_device.cuh", "zero_internal.h", "zero_tma.cuh", "zero_tma_pass.cu"),
    # the fused bfloat16 step and its replica pass (zero_kernels.cu)
    "fused-tma-bf16": ("zero_device.cuh", "zero_internal.h", "zero_tma.cuh", "zero_tma.cu", "zero_kernels.cu"),
    "fused-bf16": ("zero_device.cuh", "zero_internal.h", "zero_kernels.cu"),
}


def kernel_sha(variant):
    """Hash of the device sources the variant's step kernel is built from."""
    h = hashlib.sha256()
    for name in KERNEL_FILES[variant]:
        with open(os.path.join(CSRC, name), "rb") as f:
            h.update(name.encode() + b"\0" + f.read())
    return h.hexdigest()


def recorded_traffic(wl_name, variant):
    """DRAM bytes per launch of the dominant kernel from the committed ncu
    summary, if it was taken on the current kernel source."""
    if variant not in KERNEL_FILES:
        return None
    path = os.path.join(ROOT, "profiles", f"ncu_step_{wl_name}_{variant}.md")
    try:
        txt = open(path).read()
    except OSError:
        return None
    m = re.search(r"traffic_bytes_per_launch:\s*([0-9.eE+]+)", txt)
    h = re.search(r"kernel_source_sha256:\s*([0-9a-f]{64})", txt)
    if not m or not h or h.group(1) != kernel_sha(variant):
        return None
    return float(m.group(1))


class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.proc = None
        try:
            import torch
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            gid = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={gid}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=10)
        except Exception:
            self.proc.kill()
            return None
        rows = [r for r in csv.reader(io.StringIO(out)) if len(r) >= 8]
        if not rows:
            return None
        sm = [float(r[0]) for r in rows if r[0].strip().replace(".", "").isdigit()]
        mx = [float(r[1]) for r in rows if r[1].strip().replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[4:8]) if v.strip() == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons, "samples": len(rows)}


def cpu_info():
    model = ""
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                model = line.split(":", 1)[1].strip()
                break
    except OSError:
        pass
    return model, os.cpu_count()


# ---------------------------------------------------------------- ranks
def max_over_ranks(x: float, device: str) -> float:
    """The largest x over all ranks (the device time of the slowest rank);
    x itself without a multi-rank process group."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_value(elements_per_rank: int, steps: int, world: int, max_ms: float) -> float:
    """Gparams/s of the whole job: every rank updates elements_per_rank per
    step (weak scaling), timed by the slowest rank."""
    return world * elements_per_rank * steps / (max_ms / 1e3) / 1e9


# ---------------------------------------------------------------- oracle leg
def oracle_sample_step(wl, n_s, step, state):
    """One oracle step over the first n_s owned elements of the workload (the
    sample): the stage's own partitioned emulation with the same Nd. Returns
    CPU seconds of the oracle call alone."""
    import numpy as np

    from oracle import zero_ref as Z
    from zero_partitioned_mixed_02_b200 import synth as S

    b0, _ = owned_range(wl)
    hp = Z.hyper(**wl.hyper)
    if state.get("bf16"):
        # bfloat16 without master: the definition on the sample (ZeRO does not
        # change the math), gradients rounded to bfloat16 from the generator
        gs = [Z.bf16_from_f32(S.host_f32(n_s, b0, S.key(wl.seed, S.STREAM_GRAD, step, k), wl.grad))
              for k in range(wl.nd)]
        if state.get("w16") is None:
            w0 = S.host_f32(n_s, b0, S.key(wl.seed, S.STREAM_MASTER, 0, 0), wl.master)
            state["w16"] = Z.bf16_from_f32(w0)
            state["m"], state["v"], state["t"] = np.zeros(n_s, np.float32), np.zeros(n_s, np.float32), 0
        t0 = time.perf_counter()
        _, state["t"] = Z.bf16_step(gs, state["w16"], state["m"], state["v"], wl.loss_scale, hp, state["t"])
        return time.perf_counter() - t0
    gs = [S.host_f16_bits(n_s, b0, S.key(wl.seed, S.STREAM_GRAD, step, k), wl.grad)
          for k in range(wl.nd)]
    if state.get("w") is None:
        w0 = S.host_f32(n_s, b0, S.key(wl.seed, S.STREAM_MASTER, 0, 0), wl.master)
        if wl.stage <= 2 and wl.rank_view < 0:
            parts = [Z.partition(n_s, wl.nd, r) for r in range(wl.nd)]
            state["w"] = [w0[b:e].copy() for b, e in parts]
            state["m"] = [np.zeros(e - b, np.float32) for b, e in parts]
            state["v"] = [np.zeros(e - b, np.float32) for b, e in parts]
            state["p"] = [Z.f16_from_f32(w0) for _ in range(wl.nd)]
        elif wl.stage == 3:
            numel, left = [], n_s
            for n, _ in wl.tensors:
                take = min(n, left)
                if take <= 0:
                    break
                numel.append(take)
                left -= take
            state["numel"] = numel
            offs = np.concatenate([[0], np.cumsum(numel)])
            state["w"] = []
            for r in range(wl.nd):
                pieces = [w0[offs[t] + b: offs[t] + e]
                          for t, n in enumerate(numel) for b, e in [Z.chunk(n, wl.nd, r)]]
                state["w"].append(np.concatenate(pieces).astype(np.float32))
            state["m"] = [np.zeros_like(x) for x in state["w"]]
            state["v"] = [np.zeros_like(x) for x in state["w"]]
            state["p"] = [Z.f16_from_f32(x) for x in state["w"]]
        else:
            state["w"], state["m"], state["v"] = w0, np.zeros(n_s, np.float32), np.zeros(n_s, np.float32)
            state["p"] = np.zeros(n_s, np.uint16)
        state["t"] = 0
    t0 = time.perf_counter()
    if wl.stage <= 2 and wl.rank_view < 0:
        _, state["t"] = Z.zero12_step(n_s, gs, state["w"], state["m"], state["v"], state["p"],
                                      wl.loss_scale, hp, state["t"])
    elif wl.stage == 3:
        _, state["t"] = Z.zero3_step(state["numel"], gs, state["w"], state["m"], state["v"],
                                     state["p"], wl.loss_scale, hp, state["t"])
    else:
        _, state["t"] = Z.dp_step(gs, state["w"], state["m"], state["v"], state["p"],
                                  wl.loss_scale, hp, state["t"])
    return time.perf_counter() - t0


def calibrate_sample(wl, seconds, bf16=False):
    n0 = 1 << 17
    dt = oracle_sample_step(wl, n0, 0, {"bf16": bf16})
    rate = n0 / max(dt, 1e-6)
    b0, e0 = owned_range(wl)
    return int(max(4096, min(e0 - b0, rate * seconds)))


def cpu_baseline(wl, seconds, bf16=False):
    n_s = calibrate_sample(wl, seconds, bf16)
    dt = oracle_sample_step(wl, n_s, 0, {"bf16": bf16})
    model, ncpu = cpu_info()
    return {"value": n_s / dt / 1e9, "unit": UNIT, "cores": 1, "kind": "oracle",
            "sample": f"first {n_s} of the workload's {owned_range(wl)[1] - owned_range(wl)[0]} "
                      f"elements, Nd={wl.nd}, stage {wl.stage}, one step, single thread",
            "seconds": dt, "host_cpu": model, "host_cpus": ncpu}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    wl = workload(args.workload)
    budget = 150.0  # seconds of CPU for warm-up + timed steps
    per_step = budget / max(1, args.steps + args.warmup)
    bf16 = args.precision == "bf16"
    n_s = calibrate_sample(wl, per_step, bf16)
    state = {"bf16": bf16}
    for i in range(args.warmup):
        oracle_sample_step(wl, n_s, i, state)
    times = [oracle_sample_step(wl, n_s, args.warmup + i, state) for i in range(args.steps)]
    total = sum(times)
    value = n_s * args.steps / total / 1e9
    model, ncpu = cpu_info()
    sample = (f"first {n_s} elements of the workload per step, Nd={wl.nd}, stage {wl.stage}, "
              f"{'bfloat16 without master, ' if bf16 else ''}single thread")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * total / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {**config_of(wl, args.variant), "precision": args.precision},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle",
                         "sample": sample, "host_cpu": model, "host_cpus": ncpu},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def config_of(wl, variant):
    n, floor, _, gathers = algorithmic_bytes(wl, variant)
    return {"workload": wl.name, "psi": wl.psi, "nd": wl.nd, "stage": wl.stage,
            "rank_view": wl.rank_view, "variant": variant, "elements_updated": n,
            "loss_scale": wl.loss_scale, "weight_decay": wl.weight_decay,
            "l2": f"inputs larger than L2: {(floor + gathers) / 1e9:.1f} GB moved per step, no flush",
            "parallelism": "replicas (Nd virtual ranks emulated per GPU)"}


# ---------------------------------------------------------------- GPU leg
SPEC_HBM_GBS = 8000.0  # the B200's HBM3e specification (context beside the measured peak)
# the configurations with psi >= 1B that a default single-GPU run also times,
# beside the headline workload
PER_CONFIG = ("7.5b-rank-view", "llama-2.7b")
PER_CONFIG_E2E_STEPS = 3


def run_ours(args):
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local))

    line, wl, bf16 = measure(args, args.workload, args.variant, args.e2e_steps, world, rank, local,
                             prefetch=args.prefetch)
    if (world == 1 and not args.no_per_config and args.precision == "fp16" and not args.async_steps
            and args.workload in PER_CONFIG + ("gpt2-1.5b",)):
        # the other large configurations, one after the other in the same run
        # (each allocates its own buffers after the previous one's are freed)
        line["per_config"] = {}
        for name in PER_CONFIG:
            if name == args.workload:
                continue
            torch.cuda.empty_cache()
            if hasattr(torch._C, "_host_emptyCache"):
                torch._C._host_emptyCache()  # the previous end-to-end leg's pinned buffers
            sub, _, _ = measure(args, name, args.variant, min(args.e2e_steps, PER_CONFIG_E2E_STEPS), world,
                                rank, local, prefetch=False, with_stream_copy=False)
            line["per_config"][name] = {k: sub[k] for k in (
                "value", "unit", "ms_per_step", "config", "hbm_gbs", "roofline", "gpu_launches", "clocks",
                "gathers", "e2e") if k in sub}
            torch.cuda.empty_cache()

    if rank == 0 and not args.no_cpu_baseline and world == 1:
        line["cpu_baseline"] = cpu_baseline(wl, args.cpu_seconds, bf16)
    if world > 1:
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


def measure(args, wl_name, variant_name, e2e_steps, world, rank, local, prefetch=False, with_stream_copy=True):
    """Time one workload on this GPU: warm-up steps, then args.steps timed
    steps (and on stage 3 the forward + backward layer gathers of each step),
    the dominant kernel's roofline, and the end-to-end leg. Every buffer is
    freed when it returns. Returns (line, workload, bf16)."""
    import torch
    import torch.distributed as dist

    from zero_partitioned_mixed_02_b200 import _abi as A
    from zero_partitioned_mixed_02_b200 import synth as S

    wl = workload(wl_name)
    bf16 = args.precision == "bf16"
    if bf16 and variant_name in ("fused", "fused-tma") and not bf16_fused_eligible(wl):
        variant_name = "two-pass-tma"  # without a master and a second replica: the two-pass step
    variant = {"fused": A.ZERO_VARIANT_FUSED, "two-pass": A.ZERO_VARIANT_TWO_PASS,
               "fused-tma": A.ZERO_VARIANT_FUSED_TMA, "two-pass-tma": A.ZERO_VARIANT_TWO_PASS_TMA}[variant_name]
    two_pass = variant_name.startswith("two-pass")
    cfg = A.Config(wl.psi, wl.nd, wl.stage, rank_view=wl.rank_view, variant=variant,
                   tensors=wl.tensors,
                   precision=A.ZERO_PRECISION_BF16 if bf16 else A.ZERO_PRECISION_FP16)
    L = A.zero_state_bytes(cfg)
    b0, e0 = owned_range(wl)
    n_own = e0 - b0
    stream = torch.cuda.current_stream()
    s = stream.cuda_stream
    ws = torch.empty(L.workspace_bytes, dtype=torch.uint8, device="cuda")
    m_init = torch.empty(n_own, dtype=torch.float32, device="cuda")
    S.fill_f32(m_init.data_ptr(), n_own, b0, S.key(wl.seed, S.STREAM_MASTER, 0, 0), wl.master, s)
    bufs = []
    if wl.stage <= 2:
        bufs = [torch.empty(wl.psi, dtype=torch.int16, device="cuda")
                for _ in range(wl.nd if wl.rank_view < 0 else 1)]
    grads = [torch.empty(n_own, dtype=torch.int16, device="cuda") for _ in range(wl.nd)]
    for k in range(wl.nd):
        if bf16:
            # the generator's binary32 values rounded to bfloat16 (nearest even)
            tmp = torch.empty(n_own, dtype=torch.float32, device="cuda")
            S.fill_f32(tmp.data_ptr(), n_own, b0, S.key(wl.seed, S.STREAM_GRAD, 0, k), wl.grad, s)
            grads[k].copy_(tmp.to(torch.bfloat16).view(torch.int16))
            del tmp
        else:
            S.fill_f16(grads[k].data_ptr(), n_own, b0, S.key(wl.seed, S.STREAM_GRAD, 0, k), wl.grad, s)
    h = A.zero_init(cfg, ws.data_ptr(), L.workspace_bytes, m_init.data_ptr(),
                    [b.data_ptr() for b in bufs] if bufs else None, s)
    del m_init
    gptrs = [g.data_ptr() for g in grads]
    hp = A.zero_hyper(wl.lr, wl.beta1, wl.beta2, wl.eps, wl.weight_decay)
    gather_out = None
    if wl.stage == 3:
        gather_out = torch.empty(L.transient_bytes // 2, dtype=torch.int16, device="cuda")
    order = (list(range(L.n_units)) + list(reversed(range(L.n_units)))) if wl.stage == 3 else []

    kernel_events = []
    gather_events = []
    if args.async_steps:
        # steps enqueued back to back; the loss scale is dynamic on the device
        sc = A.zero_scaler(wl.loss_scale, 2.0, 0.5, 2000)
        A.zero_async_begin(h, gptrs, sc, wl.beta1, wl.beta2, s)

    def one_step(timed):
        if args.async_steps:
            if timed:
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
            A.zero_step_async(h, hp, s)
            if timed:
                b.record(stream)
                kernel_events.append((a, b))
            for u in order:
                A.zero_gather_layer(h, u, gather_out.data_ptr(), s)
            return
        if timed:
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
        A.zero_step_launch(h, gptrs, wl.loss_scale, hp, s)
        if timed:
            b.record(stream)
            kernel_events.append((a, b))
        rc = A.zero_step_commit(h, s)
        if rc != A.ZERO_OK:
            raise RuntimeError("unexpected skip in the benchmark workload")
        if order:
            if timed:
                c, d = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                c.record(stream)
            for u in order:
                A.zero_gather_layer(h, u, gather_out.data_ptr(), s)
            if timed:
                d.record(stream)
                gather_events.append((c, d))

    for _ in range(args.warmup):
        one_step(False)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks = ClockSampler(local) if rank == 0 else None
    time.sleep(0.3 if clocks else 0)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    t0.record(stream)
    for _ in range(args.steps):
        one_step(True)
    t1.record(stream)
    torch.cuda.synchronize()
    clock_info = clocks.stop() if clocks else None
    if args.async_steps:
        st = A.zero_async_end(h, s)
        if st.skipped:
            raise RuntimeError("unexpected skip in the benchmark workload")
    total_ms = max_over_ranks(t0.elapsed_time(t1), "cuda")
    kern_ms = [a.elapsed_time(b) for a, b in kernel_events]
    if world > 1:
        dist.barrier()

    n, floor, per_launch, gathers = algorithmic_bytes(wl, variant_name, bf16)
    launches_per_step = (2 if two_pass else 1) + len(order)
    if args.async_steps:  # + the conditional roll-back or replica pass (fused variants) and the commit kernel
        launches_per_step += 1 if two_pass else 2
    elif bf16 and not two_pass:  # + the replica pass the commit launches
        launches_per_step += 1
    step_s = total_ms / 1e3 / args.steps
    value = whole_job_value(n, args.steps, world, total_ms)
    peak, peak_src = measured_peak()
    # dominant kernel: the step kernel (both kernels of the two-pass variant
    # timed together); the fused bfloat16 step's replica pass runs in the
    # commit, outside the synchronous events (inside the asynchronous ones)
    k_s = statistics.mean(kern_ms) / 1e3
    dom_bytes = floor
    if bf16 and not two_pass:
        dom_bytes = per_launch["step_kernel<fused,bf16>"] + (per_launch["replica_kernel"] if args.async_steps else 0)
    achieved = dom_bytes / k_s / 1e9
    # a TMA variant on an ineligible layout (Nd > 16) runs the plain kernel:
    # its traffic record is the plain variant's
    ran = variant_name if (A.zero_uses_tma(h) or "tma" not in variant_name) else variant_name.replace("-tma", "")
    traffic = recorded_traffic(wl_name, ran + ("-bf16" if bf16 else ""))
    codec = ",bf16" if bf16 else ""
    if not two_pass and bf16:
        kname = ("step_tma_kernel<bf16>" if A.zero_uses_tma(h) else "step_kernel<fused,bf16>") + \
            (" + replica_kernel" if args.async_steps else "")
    elif two_pass and A.zero_uses_tma(h):
        kname = f"pass_tma_kernel<reduce{codec}>+<update{codec}>"
    elif two_pass:
        kname = f"step_kernel<reduce{codec}>+<update{codec}>"
    elif A.zero_uses_tma(h):
        kname = "step_tma_kernel"
    else:
        kname = "step_kernel<fused>"

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": config_of(wl, variant_name),
        "hbm_gbs": (floor + gathers) / step_s / 1e9,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": traffic, "kernel": kname,
                     "algorithmic_bytes_per_launch": dom_bytes,
                     "kernel_ms": statistics.mean(kern_ms), "peak_source": peak_src,
                     "spec_gbs": SPEC_HBM_GBS, "spec_frac": achieved / SPEC_HBM_GBS},
        "mode": "async" if args.async_steps else "sync",
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clock_info,
    }
    # this library's copy kernel on 4 GB, after the timed region (context for
    # the measured peak, which stays the denominator)
    if with_stream_copy:
        line["stream_copy"] = {"kernel": "zero_stream_copy", "bytes": 1 << 32, "gbs": stream_copy_gbs(),
                               "frac_of_peak": None}
        line["stream_copy"]["frac_of_peak"] = line["stream_copy"]["gbs"] / peak
    if gather_events:
        g_ms = statistics.mean(a.elapsed_time(b) for a, b in gather_events)
        g_gbs = gathers / (g_ms / 1e3) / 1e9
        line["gathers"] = {"per_step_ms": g_ms, "launches_per_step": len(order),
                           "bytes_per_step": gathers, "achieved_gbs": g_gbs,
                           "frac": g_gbs / peak, "spec_frac": g_gbs / SPEC_HBM_GBS}

    if prefetch and wl.stage == 3:
        line["prefetch"] = prefetch_demo(h, L, order, gather_out)

    # ---- end to end through the public API from pinned host buffers ----
    if not args.no_e2e and e2e_steps > 0:
        line["e2e"] = e2e(args, wl, h, grads, gptrs, bufs, ws, L, hp, order, gather_out, world, e2e_steps)
    A.zero_destroy(h)
    return line, wl, bf16


def prefetch_demo(h, L, order, gather_out, reps=5):
    """Layer gathers of a forward + backward pass, each unit consumed by a
    stand-in GEMM (tokens x d times the unit's first d x d weights), one after
    the other on one stream vs with the next unit prefetched on a side stream
    into a second transient buffer. Returns times and the measured peak."""
    import torch

    from zero_partitioned_mixed_02_b200 import _abi as A
    from zero_partitioned_mixed_02_b200.prefetch import LayerPrefetcher

    s = torch.cuda.current_stream()
    d, tokens = 2560, 8192
    x = torch.randn(tokens, d, dtype=torch.float16, device="cuda")

    def consume(w):
        return torch.mm(x, w[: d * d].view(torch.float16).view(d, d))

    def timed(fn):
        fn()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(s)
        for _ in range(reps):
            fn()
        b.record(s)
        torch.cuda.synchronize()
        return a.elapsed_time(b) / reps

    def sequential():
        for u in order:
            A.zero_gather_layer(h, u, gather_out.data_ptr(), s.cuda_stream)
            consume(gather_out)

    def gathers_only():
        for u in order:
            A.zero_gather_layer(h, u, gather_out.data_ptr(), s.cuda_stream)

    def gemms_only():
        for _ in order:
            consume(gather_out)

    torch.cuda.synchronize()
    torch.cuda.reset_peak_memory_stats()
    base = torch.cuda.memory_allocated()
    pf = LayerPrefetcher(h, L, s)
    pf_hi = LayerPrefetcher(h, L, s, priority=-1)  # side stream at high priority

    def prefetched():
        for _, w in pf.walk(order):
            consume(w)

    def prefetched_hi():
        for _, w in pf_hi.walk(order):
            consume(w)

    out = {"units": len(order), "tokens": tokens, "d": d,
           "gathers_only_ms": timed(gathers_only), "gemms_only_ms": timed(gemms_only),
           "sequential_ms": timed(sequential), "prefetched_ms": timed(prefetched),
           "prefetched_high_priority_ms": timed(prefetched_hi),
           "transient_bytes": L.transient_bytes, "prefetch_transient_bytes": pf.peak_bytes}
    out["measured_peak_extra_bytes"] = torch.cuda.max_memory_allocated() - base
    hidden = out["sequential_ms"] - out["prefetched_ms"]
    out["gather_time_hidden_frac"] = hidden / out["gathers_only_ms"]
    out["gather_time_hidden_frac_high_priority"] = (
        out["sequential_ms"] - out["prefetched_high_priority_ms"]) / out["gathers_only_ms"]
    return out


def e2e(args, wl, h, grads, gptrs, bufs, ws, L, hp, order, gather_out, world, steps):
    import psutil
    import torch
    import torch.distributed as dist

    from zero_partitioned_mixed_02_b200 import _abi as A

    n_own = grads[0].numel()
    if wl.stage <= 2 and wl.rank_view >= 0:
        b0, e0 = owned_range(wl)
        result = bufs[0][b0:e0]  # the step's result: the new fp16 partition of this rank
    elif wl.stage <= 2:
        result = bufs[0]  # the step's result: one rank's all-gathered fp16 parameters
    else:
        result = ws[L.off_shard16: L.off_shard16 + 2 * L.state_elems].view(torch.int16)
    need = (len(grads) * n_own + result.numel()) * 2
    avail = psutil.virtual_memory().available
    # every rank on this node pins its own copies at the same time
    local_ranks = int(os.environ.get("LOCAL_WORLD_SIZE", str(world)))
    ok = need * local_ranks <= 0.6 * avail
    if world > 1:  # every rank takes the same decision (the steps below hold collectives)
        flag = torch.tensor([1 if ok else 0], device="cuda")
        dist.all_reduce(flag, op=dist.ReduceOp.MIN)
        ok = bool(flag.item())
    if not ok:
        return {"value": None, "unit": UNIT,
                "unavailable": f"needs {need / 1e9:.1f} GB pinned host memory per rank x {local_ranks} "
                               f"ranks, {avail / 1e9:.1f} GB available"}
    s = torch.cuda.current_stream()
    side = torch.cuda.Stream()  # device->host reads of the result
    up = torch.cuda.Stream()    # host->device uploads of the gradients
    host_g = [torch.empty(n_own, dtype=torch.int16, pin_memory=True) for _ in grads]
    for hg, g in zip(host_g, grads):
        hg.copy_(g)
    host_out = torch.empty(result.numel(), dtype=torch.int16, pin_memory=True)
    # two device gradient sets: step k reads set k % 2 while the inputs of
    # step k + 1 travel into the other one (every step's inputs still cross
    # the link inside the timed region)
    try:
        sets = [grads, [torch.empty_like(g) for g in grads]]
        pipelined = True
    except torch.cuda.OutOfMemoryError:  # one set: each upload waits for the step before
        sets = [grads, grads]
        pipelined = False
    ptrs = [[g.data_ptr() for g in x] for x in sets]
    uploaded = [None, None]  # upload of each set done
    used = [None, None]      # last step that read each set done
    read_done = None

    def upload(k):
        i = k % 2
        if used[i] is not None:
            up.wait_event(used[i])
        with torch.cuda.stream(up):
            for g, hg in zip(sets[i], host_g):
                g.copy_(hg, non_blocking=True)
        uploaded[i] = torch.cuda.Event()
        uploaded[i].record(up)

    def step(k, last):
        # enqueue the next step's upload first: it runs while this step's
        # kernels run and the last step's result is read back
        nonlocal read_done
        i = k % 2
        if pipelined and k + 1 <= last:
            upload(k + 1)
        s.wait_event(uploaded[i])
        if read_done is not None:
            s.wait_event(read_done)  # the result buffer is free again
        rc = A.zero_step(h, ptrs[i], wl.loss_scale, hp, s.cuda_stream)
        if rc != A.ZERO_OK:
            raise RuntimeError("unexpected skip")
        for u in order:
            A.zero_gather_layer(h, u, gather_out.data_ptr(), s.cuda_stream)
        done = torch.cuda.Event()
        done.record(s)
        used[i] = done
        side.wait_event(done)
        with torch.cuda.stream(side):
            host_out.copy_(result, non_blocking=True)
        read_done = torch.cuda.Event()
        read_done.record(side)
        if not pipelined and k + 1 <= last:
            upload(k + 1)  # after the step: it overwrites the gradients the step read

    upload(0)
    step(0, 0)  # warm-up
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(s)
    up.wait_event(a)
    upload(0)
    for k in range(steps):
        step(k, steps - 1)
    s.wait_event(read_done)  # the last read-back is inside the timed region
    b.record(s)
    torch.cuda.synchronize()
    ms = max_over_ranks(a.elapsed_time(b), "cuda")
    n = L.state_elems
    return {"value": whole_job_value(n, steps, world, ms), "unit": UNIT,
            "h2d_bytes_per_step": len(grads) * n_own * 2, "d2h_bytes_per_step": result.numel() * 2,
            "steps": steps, "ms_per_step": ms / steps, "pipelined": pipelined}


# ---------------------------------------------------------------- the real job
NVLINK_PEER_GBS = 770.0  # measured peer copy on this machine, per direction per GPU (nominal 900)


def zero_job_bytes(psi: int, world: int, stage: int, n_units_elems: int = 0) -> dict:
    """Bytes one rank of the real Nd = world job moves per step, for the
    slowest (first, full-length) partition P = ceil(psi / world). Stage 1/2:
    it pulls partition r of the other ranks' fp16 gradients over NVLink and
    stores the new fp16 partition into the other ranks' parameter buffers;
    its own HBM serves its gradient slice to every rank, its state, and every
    rank's store into its parameter buffer. Stage 3: the same pull of the
    gradient chunks, the fp16 shard stays local; each layer gather pulls the
    other ranks' chunks of the unit (n_units_elems: elements gathered per step
    over all units, forward and backward)."""
    P = -(-psi // world)
    remote = world - 1
    out = {"partition": P, "nvlink_in": 2 * P * remote, "nvlink_out": 0, "hbm": 0}
    if stage <= 2:
        out["nvlink_out"] = 2 * P * remote
        out["hbm"] = 2 * P * world + 24 * P + 2 * P * world
    else:
        out["hbm"] = 2 * P * world + 24 * P + 2 * P
        # gathers: (world - 1)/world of every unit's elements come from peers
        out["nvlink_in_gathers"] = 2 * n_units_elems * remote // world
    return out


def run_zero_job(args):
    """The real Nd = N job (the method across GPUs): one process per GPU,
    rank r owns partition r (stage 1/2) or chunk r of every tensor (stage 3)
    of the workload's parameter list; its step pulls the other ranks'
    gradients of that partition through peer mappings, sums them in rank order
    and runs Adam, then stores the new fp16 partition into every rank's
    parameter buffer (stage 1/2; distributed.PeerRank); the overflow decision
    is MAX-reduced between launch and commit. Timed with CUDA events on each
    rank's stream, max over ranks; whole-job Gparams/s = psi per step. Beside
    it: NCCL reduce-scatter + all-gather of the same fp16 bytes (NCCL backend
    only)."""
    from datetime import timedelta

    import torch
    import torch.distributed as dist

    from zero_partitioned_mixed_02_b200 import _abi as A
    from zero_partitioned_mixed_02_b200 import synth as S
    from zero_partitioned_mixed_02_b200.distributed import PeerRank, device_barrier

    world = int(os.environ["WORLD_SIZE"])
    rank = int(os.environ["RANK"])
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dev = local % max(torch.cuda.device_count(), 1)
    torch.cuda.set_device(dev)
    if args.backend == "nccl":
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", dev))
    else:
        dist.init_process_group("gloo", timeout=timedelta(seconds=120))
    wl = workload(args.workload)
    if wl.rank_view >= 0:
        raise SystemExit("the real job runs a full-model workload (not the rank view)")
    variant = {"fused": A.ZERO_VARIANT_FUSED, "two-pass": A.ZERO_VARIANT_TWO_PASS,
               "fused-tma": A.ZERO_VARIANT_FUSED_TMA, "two-pass-tma": A.ZERO_VARIANT_TWO_PASS_TMA}[args.variant]
    stream = torch.cuda.current_stream()
    s = stream.cuda_stream
    psi, stage = wl.psi, wl.stage
    grad = torch.empty(psi, dtype=torch.int16, device="cuda")
    S.fill_f16(grad.data_ptr(), psi, 0, S.key(wl.seed, S.STREAM_GRAD, 0, rank), wl.grad, s)
    P = -(-psi // world)
    b, e = (min(rank * P, psi), min(rank * P + P, psi)) if stage <= 2 else (0, psi)
    m_init = torch.empty(e - b, dtype=torch.float32, device="cuda")
    S.fill_f32(m_init.data_ptr(), e - b, b, S.key(wl.seed, S.STREAM_MASTER, 0, 0), wl.master, s)
    params = torch.empty(psi, dtype=torch.int16, device="cuda") if stage <= 2 else None
    job = PeerRank(grad, params, m_init, stage=stage, variant=variant, tensors=wl.tensors, stream=stream)
    del m_init
    hp = A.zero_hyper(wl.lr, wl.beta1, wl.beta2, wl.eps, wl.weight_decay)
    order, gather_out, gathered = [], None, 0
    if stage == 3:
        L = A.zero_state_bytes(job.cfg)
        order = list(range(L.n_units)) + list(reversed(range(L.n_units)))
        gather_out = torch.empty(L.transient_bytes // 2, dtype=torch.int16, device="cuda")
        gathered = sum(job.unit_range(u)[1] for u in order)

    step_ev, gather_ev = [], []

    def one_step(timed):
        if timed:
            a, c = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
        if job.step(wl.loss_scale, hp):
            raise RuntimeError("unexpected skip in the benchmark workload")
        if timed:
            c.record(stream)
            step_ev.append((a, c))
        if order:
            if timed:
                g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                g0.record(stream)
            for u in order:
                job.gather(u, gather_out)
            if timed:
                g1.record(stream)
                gather_ev.append((g0, g1))

    for _ in range(args.warmup):
        one_step(False)
    torch.cuda.synchronize()
    dist.barrier()
    clocks = ClockSampler(dev) if rank == 0 else None
    time.sleep(0.3 if clocks else 0)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(args.steps):
        one_step(True)
    t1.record(stream)
    torch.cuda.synchronize()
    clock_info = clocks.stop() if clocks else None
    dev_str = "cuda" if args.backend == "nccl" else "cpu"
    total_ms = max_over_ranks(t0.elapsed_time(t1), dev_str)
    step_ms = max_over_ranks(statistics.mean(a.elapsed_time(c) for a, c in step_ev), dev_str)
    g_ms = max_over_ranks(statistics.mean(a.elapsed_time(c) for a, c in gather_ev), dev_str) if gather_ev else None

    by = zero_job_bytes(psi, world, stage, gathered)
    nv_dir = max(by["nvlink_in"], by["nvlink_out"])
    nv_gbs = nv_dir / (step_ms / 1e3) / 1e9
    peak, peak_src = measured_peak()
    line = {
        "metric": METRIC, "value": psi * args.steps / (total_ms / 1e3) / 1e9, "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": total_ms / args.steps,
        "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic",
        "config": {"workload": wl.name, "psi": psi, "nd": world, "stage": stage, "variant": args.variant,
                   "elements_updated": psi, "partition": P, "loss_scale": wl.loss_scale,
                   "weight_decay": wl.weight_decay, "backend": args.backend,
                   "l2": "inputs larger than L2, no flush",
                   "parallelism": f"zero-dp{world}: one partition per GPU, the reduce-scatter and "
                                  f"all-gather fused into the step over peer memory"},
        "roofline": {"bound": "nvlink", "achieved": nv_gbs, "peak": NVLINK_PEER_GBS, "unit": "GB/s",
                     "frac": nv_gbs / NVLINK_PEER_GBS, "traffic": None, "kernel": "rank step",
                     "algorithmic_bytes_per_launch": nv_dir, "kernel_ms": step_ms,
                     "peak_source": "measured peer copy on this pool, per direction",
                     "hbm_bytes_per_rank": by["hbm"],
                     "hbm_gbs": by["hbm"] / (step_ms / 1e3) / 1e9, "hbm_peak": peak,
                     "hbm_peak_source": peak_src},
        "gpu_launches": ((2 if args.variant.startswith("two-pass") else 1) + len(order)) * args.steps,
        "clocks": clock_info,
    }
    if g_ms is not None:
        line["gathers"] = {"per_step_ms": g_ms, "launches_per_step": len(order),
                           "nvlink_in_bytes_per_rank": by["nvlink_in_gathers"],
                           "nvlink_gbs": by["nvlink_in_gathers"] / (g_ms / 1e3) / 1e9}

    if args.backend == "nccl" and stage <= 2:
        # NCCL's reduce-scatter + all-gather of the same fp16 bytes (no Adam,
        # fp16 sums in NCCL's order): what the fused step replaces
        pad = P * world
        g16 = torch.zeros(pad, dtype=torch.float16, device="cuda")
        g16[:psi].copy_(grad.view(torch.float16))
        part = torch.empty(P, dtype=torch.float16, device="cuda")
        full = torch.empty(pad, dtype=torch.float16, device="cuda")

        def rs_ag():
            dist.reduce_scatter_tensor(part, g16)
            dist.all_gather_into_tensor(full, part)

        for _ in range(max(args.warmup, 1)):
            rs_ag()
        torch.cuda.synchronize()
        dist.barrier()
        a, c = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(args.steps):
            rs_ag()
        c.record(stream)
        torch.cuda.synchronize()
        n_ms = max_over_ranks(a.elapsed_time(c) / args.steps, "cuda")
        line["nccl_rs_ag"] = {"ms_per_step": n_ms, "bytes_per_rank_per_direction": 2 * P * (world - 1),
                              "gbs_per_direction": 2 * P * (world - 1) / (n_ms / 1e3) / 1e9,
                              "vs_rank_step": n_ms / step_ms}
        del g16, part, full

    if not args.no_e2e and args.e2e_steps > 0:
        # end to end: every step uploads this rank's gradient from pinned host
        # memory and reads back the step's result (this rank's new fp16
        # partition, or its shard)
        host_g = torch.empty(psi, dtype=torch.int16, pin_memory=True)
        host_g.copy_(grad)
        res = params[b:e] if stage <= 2 else job.workspace[
            A.zero_state_bytes(job.cfg).off_shard16:].view(torch.int16)[: A.zero_state_bytes(job.cfg).state_elems]
        host_out = torch.empty(res.numel(), dtype=torch.int16, pin_memory=True)
        device_barrier(stream)
        a, c = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(args.e2e_steps):
            grad.copy_(host_g, non_blocking=True)
            if job.step(wl.loss_scale, hp):
                raise RuntimeError("unexpected skip")
            for u in order:
                job.gather(u, gather_out)
            host_out.copy_(res, non_blocking=True)
        c.record(stream)
        torch.cuda.synchronize()
        e_ms = max_over_ranks(a.elapsed_time(c), dev_str)
        line["e2e"] = {"value": psi * args.e2e_steps / (e_ms / 1e3) / 1e9, "unit": UNIT,
                       "h2d_bytes_per_step": 2 * psi, "d2h_bytes_per_step": 2 * res.numel(),
                       "steps": args.e2e_steps, "ms_per_step": e_ms / args.e2e_steps,
                       "per_rank": True}
    job.close()
    dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


def host_copy_gbs(threads, n_bytes=1 << 31, reps=5):
    """Host memory bandwidth reference for the offloaded update: a torch copy
    of n_bytes on `threads` threads, read + written bytes per second (best of
    reps)."""
    import torch

    old = torch.get_num_threads()
    torch.set_num_threads(threads)
    a = torch.ones(n_bytes // 4, dtype=torch.float32)
    b = torch.empty_like(a)
    b.copy_(a)
    best = float("inf")
    for _ in range(reps):
        t0 = time.perf_counter()
        b.copy_(a)
        best = min(best, time.perf_counter() - t0)
    torch.set_num_threads(old)
    return 2 * n_bytes / best / 1e9


def run_offload(args):
    """The offloaded step on the workload: fp32 master/m/v in host memory, Adam
    on the host cores, reduce and fp16 write-back on the GPU, chunks pipelined
    over PCIe. Timed with CUDA events on the caller's stream, which bracket
    every device and host part of each step (the device work of a step waits
    for the host update of its chunks)."""
    import numpy as np
    import torch

    from zero_partitioned_mixed_02_b200 import _abi as A
    from zero_partitioned_mixed_02_b200 import synth as S

    if int(os.environ.get("WORLD_SIZE", "1")) > 1:
        raise SystemExit("--offload runs on one GPU")
    torch.cuda.set_device(0)
    wl = workload(args.workload)
    cfg = A.Config(wl.psi, wl.nd, wl.stage, rank_view=wl.rank_view, tensors=wl.tensors)
    L = A.zero_offload_bytes(cfg, args.offload_chunk)
    threads = args.offload_threads or len(os.sched_getaffinity(0))
    threads = max(1, min(threads, 256))
    b0, e0 = owned_range(wl)
    n_own = e0 - b0
    stream = torch.cuda.current_stream()
    s = stream.cuda_stream
    m_dev = torch.empty(n_own, dtype=torch.float32, device="cuda")
    S.fill_f32(m_dev.data_ptr(), n_own, b0, S.key(wl.seed, S.STREAM_MASTER, 0, 0), wl.master, s)
    master_init = m_dev.cpu().numpy()
    del m_dev
    E = L.state_elems
    state = np.empty(3 * E, np.float32)
    dws = torch.empty(L.device_bytes, dtype=torch.uint8, device="cuda")
    staging = torch.empty(L.host_staging_bytes, dtype=torch.uint8, pin_memory=True)
    if wl.stage <= 2:
        bufs = [torch.empty(wl.psi, dtype=torch.int16, device="cuda")
                for _ in range(wl.nd if wl.rank_view < 0 else 1)]
    else:
        bufs = [torch.empty(E, dtype=torch.int16, device="cuda")]
    grads = [torch.empty(n_own, dtype=torch.int16, device="cuda") for _ in range(wl.nd)]
    for k in range(wl.nd):
        S.fill_f16(grads[k].data_ptr(), n_own, b0, S.key(wl.seed, S.STREAM_GRAD, 0, k), wl.grad, s)
    t_init = time.perf_counter()
    h = A.zero_offload_init(cfg, args.offload_chunk, dws.data_ptr(), L.device_bytes, staging.data_ptr(),
                            L.host_staging_bytes, state.ctypes.data, master_init.ctypes.data,
                            [b.data_ptr() for b in bufs], threads, s)
    t_init = time.perf_counter() - t_init
    del master_init
    gptrs = [g.data_ptr() for g in grads]
    hp = A.zero_hyper(wl.lr, wl.beta1, wl.beta2, wl.eps, wl.weight_decay)
    for _ in range(args.warmup):
        if A.zero_offload_step(h, gptrs, wl.loss_scale, hp, s) != A.ZERO_OK:
            raise RuntimeError("unexpected skip in the benchmark workload")
    torch.cuda.synchronize()
    clocks = ClockSampler(0)
    time.sleep(0.3)
    ev = []
    for _ in range(args.steps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        if A.zero_offload_step(h, gptrs, wl.loss_scale, hp, s) != A.ZERO_OK:
            raise RuntimeError("unexpected skip in the benchmark workload")
        b.record(stream)
        ev.append((a, b))
    torch.cuda.synchronize()
    clock_info = clocks.stop()
    ms = [a.elapsed_time(b) for a, b in ev]
    total_ms = sum(ms)
    A.zero_offload_destroy(h)
    host_copy = host_copy_gbs(threads)
    step_s = total_ms / 1e3 / args.steps
    Ld = A.zero_state_bytes(cfg)
    pcie = L.d2h_bytes_per_step + L.h2d_bytes_per_step
    line = {
        "metric": METRIC, "value": E * args.steps / (total_ms / 1e3) / 1e9, "unit": UNIT, "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": total_ms / args.steps,
        "ms_per_step_min": min(ms), "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32", "data": "synthetic", "mode": "offload",
        "config": {**config_of(wl, "offload"), "variant": "offload"},
        "offload": {
            "host_threads": threads, "chunk_elems": L.chunk_elems, "n_chunks": L.n_chunks,
            "slots": A.ZERO_OFFLOAD_SLOTS, "init_s": t_init,
            "d2h_bytes_per_step": L.d2h_bytes_per_step, "h2d_bytes_per_step": L.h2d_bytes_per_step,
            "pcie_gbs": pcie / step_s / 1e9,
            # host memory traffic of the update: read g, w, m, v; write w, m, v, p16
            "host_update_gbs": 30 * E / step_s / 1e9,
            "host_copy_gbs": host_copy,
            "host_update_frac_of_copy": 30 * E / step_s / 1e9 / host_copy,
            "host_state_bytes": L.host_state_bytes,
            "device_state_bytes_per_rank": L.device_state_bytes,
            "device_state_bytes_per_rank_without_offload": int(Ld.exact_bytes[wl.stage]),
        },
        "gpu_launches": (1 + 2 * L.n_chunks) * args.steps,
        "clocks": clock_info,
    }
    print(json.dumps(line), flush=True)


def main():
    args = parse_args()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if args.impl == "reference":
        run_reference(args)
    elif args.offload:
        run_offload(args)
    elif world > 1 and (args.mode or "zero") == "zero":
        run_zero_job(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
