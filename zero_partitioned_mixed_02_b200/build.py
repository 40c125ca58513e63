"""Build the package's native libraries in-tree for sm_100a.

  libzero_bounds.so   the same with the kernels' index ranges checked (debug)
  libzero.so          the ZeRO step library (csrc/*.cu and the host update
                      csrc/zero_host_adam.cpp; C ABI in include/zero.h and
                      include/zero_offload.h)
  synth/libzsynth.so  the seeded synthetic-input generator (host + device)

Flags: arithmetic is IEEE binary32 as written -- no FMA contraction
(-fmad=false), correctly rounded division and square root, no flush to zero.
``python -m zero_partitioned_mixed_02_b200.build [--force]``.
"""
from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
SYNTH = os.path.join(PKG, "synth")

LIBZERO = os.path.join(PKG, "libzero.so")
# the same library with every kernel's global index ranges checked
# (ZK_BOUNDS_CHECK): an access outside a buffer is skipped and reported as
# ZERO_ERR_INTERNAL; load it with ZERO_LIBZERO=<path> to run a test suite on it
LIBZERO_DEBUG = os.path.join(PKG, "libzero_bounds.so")
LIBSYNTH = os.path.join(SYNTH, "libzsynth.so")
PTXAS_LOG = os.path.join(PKG, "libzero.ptxas.txt")

NVCC = os.environ.get("NVCC", "nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
COMMON = [*ARCH, "-lineinfo", "-O3", "-std=c++17", "-shared", "-fmad=false", "-ftz=false",
          "-prec-div=true", "-prec-sqrt=true", "-Xcompiler", "-fPIC,-ffp-contract=off"]

ZERO_SOURCES = [os.path.join(CSRC, "zero_abi.cu"), os.path.join(CSRC, "zero_kernels.cu"),
                os.path.join(CSRC, "zero_static.cu"), os.path.join(CSRC, "zero_tma.cu"),
                os.path.join(CSRC, "zero_offload.cu"), os.path.join(CSRC, "zero_tma_pass.cu"),
                os.path.join(CSRC, "zero_peer.cu"), os.path.join(CSRC, "zero_gather_ranks.cu")]
HOST_ADAM = os.path.join(CSRC, "zero_host_adam.cpp")
ZERO_DEPS = ZERO_SOURCES + [HOST_ADAM, os.path.join(CSRC, "zero_host_adam.h"),
                            os.path.join(CSRC, "zero_internal.h"), os.path.join(CSRC, "zero_device.cuh"),
                            os.path.join(CSRC, "zero_layout.h"), os.path.join(CSRC, "zero_tma.cuh"),
                            os.path.join(CSRC, "zero_gather_ranks.h"), os.path.join(CSRC, "zero_pdl.cuh"),
                            os.path.join(INCLUDE, "zero.h"),
                            os.path.join(INCLUDE, "zero_offload.h"), os.path.join(INCLUDE, "zero_peer.h")]
# the host update is built twice: AVX2 + F16C, and the baseline instruction set
# (picked at run time); binary32 as written, no contraction into FMA
CXX = os.environ.get("CXX", "g++")
HOST_FLAGS = ["-O3", "-std=c++17", "-fPIC", "-fvisibility=hidden", "-ffp-contract=off", "-fno-fast-math"]
HOST_VARIANTS = {"avx2": ["-DZH_AVX2", "-mavx2", "-mf16c"], "base": []}
SYNTH_SOURCES = [os.path.join(SYNTH, "zsynth.cu")]
SYNTH_DEPS = SYNTH_SOURCES + [os.path.join(SYNTH, "zsynth.h")]


def _stale(target: str, deps: list[str]) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps + [__file__])


def _nvcc(out: str, sources: list[str], extra: list[str], log: str | None = None) -> None:
    tmp = out + f".tmp{os.getpid()}"
    cmd = [NVCC, *COMMON, *extra, "-o", tmp, *sources]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        sys.stderr.write(res.stdout + res.stderr)
        raise RuntimeError(f"nvcc failed building {os.path.basename(out)}")
    if log is not None:
        with open(log, "w") as f:
            f.write(res.stdout + res.stderr)
    os.replace(tmp, out)


def _host_objects() -> list[str]:
    objs = []
    for name, flags in HOST_VARIANTS.items():
        obj = os.path.join(PKG, f"zero_host_adam_{name}.o")
        cmd = [CXX, *HOST_FLAGS, *flags, "-I", CSRC, "-c", HOST_ADAM, "-o", obj]
        res = subprocess.run(cmd, capture_output=True, text=True)
        if res.returncode != 0:
            sys.stderr.write(res.stdout + res.stderr)
            raise RuntimeError(f"{CXX} failed building {os.path.basename(obj)}")
        objs.append(obj)
    return objs


def build(force: bool = False) -> None:
    stale = force or _stale(LIBZERO, ZERO_DEPS)
    stale_debug = force or _stale(LIBZERO_DEBUG, ZERO_DEPS)
    if stale or stale_debug:
        objs = _host_objects()
        if stale:
            _nvcc(LIBZERO, ZERO_SOURCES + objs,
                  ["-I", INCLUDE, "-I", CSRC, "-Xcompiler", "-fvisibility=hidden", "-Xptxas", "-v"],
                  log=PTXAS_LOG)
        if stale_debug:
            _nvcc(LIBZERO_DEBUG, ZERO_SOURCES + objs,
                  ["-I", INCLUDE, "-I", CSRC, "-Xcompiler", "-fvisibility=hidden", "-DZK_BOUNDS_CHECK"])
        for o in objs:
            os.remove(o)
    if force or _stale(LIBSYNTH, SYNTH_DEPS):
        _nvcc(LIBSYNTH, SYNTH_SOURCES, ["-I", SYNTH])


if __name__ == "__main__":
    build(force="--force" in sys.argv)
    print(LIBZERO)
    print(LIBSYNTH)
