"""Seeded synthetic inputs for the tests and the benchmark.

A module of its own: it generates gradients and initial master weights and
holds none of the optimizer's arithmetic. The generator (zsynth.h) is compiled
once into ``libzsynth.so`` with a host path (used for oracle inputs and sampled
checks) and a device path (full-size inputs); both give the same binary32
values. fp16 rounding is done by numpy on the host and by ``__float2half_rn``
on the device; a GPU test checks that the two agree bit for bit.
"""
from __future__ import annotations

import ctypes as C
import os

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libzsynth.so")

STREAM_GRAD = 1
STREAM_MASTER = 2

ZS_NORMAL, ZS_UNIFORM, ZS_SIGNED_MAG, ZS_NORMAL_TINY = 0, 1, 2, 3


class Dist(C.Structure):
    _fields_ = [("kind", C.c_int32), ("tiny_per_2_24", C.c_int32), ("c", C.c_float),
                ("a", C.c_float), ("b", C.c_float), ("tiny_lo", C.c_float),
                ("tiny_hi", C.c_float), ("scale", C.c_float)]


def normal(sigma: float, scale: float = 1.0) -> Dist:
    return Dist(ZS_NORMAL, 0, float(np.float32(sigma * 2.0**-24)), 0.0, 0.0, 0.0, 0.0, scale)


def uniform(a: float, b: float) -> Dist:
    return Dist(ZS_UNIFORM, 0, 0.0, a, b, 0.0, 0.0, 1.0)


def signed_mag(a: float, b: float) -> Dist:
    return Dist(ZS_SIGNED_MAG, 0, 0.0, a, b, 0.0, 0.0, 1.0)


def normal_tiny(sigma: float, tiny_frac: float, tiny_lo: float, tiny_hi: float,
                scale: float = 1.0) -> Dist:
    thr = int(round(tiny_frac * 2**24))
    return Dist(ZS_NORMAL_TINY, thr, float(np.float32(sigma * 2.0**-24)), 0.0, 0.0,
                tiny_lo, tiny_hi, scale)


_lib = None


def lib():
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is not built; run zero_partitioned_mixed_02_b200.build")
        L = C.CDLL(LIB_PATH)
        L.zsynth_key.restype = C.c_uint64
        L.zsynth_key.argtypes = [C.c_uint64] * 4
        L.zsynth_host_f32.restype = None
        L.zsynth_host_f32.argtypes = [C.c_void_p, C.c_int64, C.c_int64, C.c_uint64, C.POINTER(Dist)]
        L.zsynth_host_f32_at.restype = None
        L.zsynth_host_f32_at.argtypes = [C.c_void_p, C.c_void_p, C.c_int64, C.c_uint64,
                                         C.POINTER(Dist)]
        for name in ("zsynth_fill_f16", "zsynth_fill_f32"):
            f = getattr(L, name)
            f.restype = C.c_int
            f.argtypes = [C.c_void_p, C.c_int64, C.c_int64, C.c_uint64, C.POINTER(Dist), C.c_void_p]
        _lib = L
    return _lib


def key(seed: int, stream: int, step: int, rank: int) -> int:
    return int(lib().zsynth_key(seed, stream, step, rank))


def host_f32(n: int, index0: int, k: int, d: Dist) -> np.ndarray:
    out = np.empty(n, np.float32)
    lib().zsynth_host_f32(out.ctypes.data, n, index0, k, C.byref(d))
    return out


def host_f32_at(idx, k: int, d: Dist) -> np.ndarray:
    idx = np.ascontiguousarray(idx, dtype=np.int64)
    out = np.empty(idx.shape, np.float32)
    lib().zsynth_host_f32_at(out.ctypes.data, idx.ctypes.data, idx.size, k, C.byref(d))
    return out


def host_f16_bits(n: int, index0: int, k: int, d: Dist) -> np.ndarray:
    with np.errstate(over="ignore"):
        return host_f32(n, index0, k, d).astype(np.float16).view(np.uint16)


def host_f16_bits_at(idx, k: int, d: Dist) -> np.ndarray:
    with np.errstate(over="ignore"):
        return host_f32_at(idx, k, d).astype(np.float16).view(np.uint16)


def fill_f16(ptr: int, n: int, index0: int, k: int, d: Dist, stream: int) -> None:
    rc = lib().zsynth_fill_f16(ptr, n, index0, k, C.byref(d), stream)
    if rc != 0:
        raise RuntimeError("zsynth_fill_f16 failed")


def fill_f32(ptr: int, n: int, index0: int, k: int, d: Dist, stream: int) -> None:
    rc = lib().zsynth_fill_f32(ptr, n, index0, k, C.byref(d), stream)
    if rc != 0:
        raise RuntimeError("zsynth_fill_f32 failed")
