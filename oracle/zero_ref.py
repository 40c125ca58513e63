"""numpy/ctypes face of the C oracle (zero_ref.c).

TEST INFRASTRUCTURE: only the test suite, the package's smoke check and the
benchmark's CPU-baseline leg import this module. It never touches a GPU and
never imports the CUDA package.

fp16 arrays are passed as ``np.uint16`` bit patterns (or ``np.float16``, which
is viewed as uint16). State arrays are ``np.float32`` and are updated in place.
"""
from __future__ import annotations

import ctypes as C
from typing import Sequence

import numpy as np

from . import build as _build

_lib = C.CDLL(_build.build())

_i64, _i32, _f32 = C.c_int64, C.c_int32, C.c_float
_p = C.c_void_p
_pp = C.POINTER(C.c_void_p)


class Hyper(C.Structure):
    _fields_ = [("lr", C.c_float), ("beta1", C.c_float), ("beta2", C.c_float),
                ("eps", C.c_float), ("weight_decay", C.c_float)]


def _sig(name, res, *args):
    f = getattr(_lib, name)
    f.restype = res
    f.argtypes = list(args)
    return f


_f32_from_f16 = _sig("zr_f32_from_f16", _f32, C.c_uint16)
_f16_from_f32 = _sig("zr_f16_from_f32", C.c_uint16, _f32)
_f16_from_f64 = _sig("zr_f16_from_f64", C.c_uint16, C.c_double)
_f32_from_f16_array = _sig("zr_f32_from_f16_array", None, _p, _p, _i64)
_f16_from_f32_array = _sig("zr_f16_from_f32_array", None, _p, _p, _i64)
_direct_array = _sig("zr_direct_f16_update_array", None, _p, _p, _p, _i64)
_partition = _sig("zr_partition", None, _i64, _i32, _i32, C.POINTER(_i64), C.POINTER(_i64))
_shard_len = _sig("zr_shard_len", _i64, _i32, _p, _i32, _i32)
_bias = _sig("zr_bias_corrections", None, _f32, _f32, _i64, C.POINTER(_f32), C.POINTER(_f32))
_inv_scale = _sig("zr_inv_scale", _f32, _f32)
_dp_step = _sig("zr_dp_step", C.c_int, _i64, _i32, _pp, _p, _p, _p, _p, _f32,
                C.POINTER(Hyper), C.POINTER(_i64))
_dp_step_masked = _sig("zr_dp_step_masked", C.c_int, _i64, _i32, _pp, _p, _p, _p, _p, _f32,
                       C.POINTER(Hyper), _p, C.POINTER(_i64))
_f32_from_bf16 = _sig("zr_f32_from_bf16", _f32, C.c_uint16)
_bf16_from_f32 = _sig("zr_bf16_from_f32", C.c_uint16, _f32)
_bf16_from_f64 = _sig("zr_bf16_from_f64", C.c_uint16, C.c_double)
_f32_from_bf16_array = _sig("zr_f32_from_bf16_array", None, _p, _p, _i64)
_bf16_from_f32_array = _sig("zr_bf16_from_f32_array", None, _p, _p, _i64)
_bf16_step = _sig("zr_bf16_step", C.c_int, _i64, _i32, _pp, _p, _p, _p, _f32, C.POINTER(Hyper), _p,
                  C.POINTER(_i64))
_z12_step = _sig("zr_zero12_step", C.c_int, _i64, _i32, _pp, _pp, _pp, _pp, _pp, _f32,
                 C.POINTER(Hyper), C.POINTER(_i64))
_z3_step = _sig("zr_zero3_step", C.c_int, _i32, _p, _i32, _pp, _pp, _pp, _pp, _pp, _f32,
                C.POINTER(Hyper), C.POINTER(_i64))
_z3_gather = _sig("zr_zero3_gather", _i64, _i32, _p, _p, _i32, _i32, _pp, _p)
_formula = _sig("zr_ledger_formula", None, C.c_double, C.c_double, C.POINTER(C.c_double))
_exact = _sig("zr_ledger_exact", None, _i64, _i32, _i32, _p, C.POINTER(_i64))
_comm = _sig("zr_comm_elements", None, _i64, _i32, C.POINTER(_i64))
_scaler = _sig("zr_scaler_update", None, C.POINTER(_f32), C.POINTER(_i32), C.c_int, _f32, _f32, _i32)


def _ptr(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data


def _ptrs(arrs: Sequence[np.ndarray]):
    vals = [_ptr(a) for a in arrs]
    return (C.c_void_p * max(len(vals), 1))(*vals)


def _u16(a) -> np.ndarray:
    a = np.ascontiguousarray(a)
    if a.dtype == np.float16:
        return a.view(np.uint16)
    assert a.dtype == np.uint16, a.dtype
    return a


def hyper(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.0) -> Hyper:
    return Hyper(lr, beta1, beta2, eps, weight_decay)


# ---- conversions ----------------------------------------------------------
def f32_from_f16(h) -> np.ndarray:
    h = _u16(h)
    out = np.empty(h.shape, np.float32)
    _f32_from_f16_array(_ptr(h), _ptr(out), h.size)
    return out


def f16_from_f32(x) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, np.uint16)
    _f16_from_f32_array(_ptr(x), _ptr(out), x.size)
    return out


def f16_from_f64_scalar(x: float) -> int:
    return int(_f16_from_f64(float(x)))


def direct_f16_update(w16, dw) -> np.ndarray:
    w16 = _u16(w16)
    dw = np.ascontiguousarray(dw, dtype=np.float32)
    out = np.empty(w16.shape, np.uint16)
    _direct_array(_ptr(w16), _ptr(dw), _ptr(out), w16.size)
    return out


# ---- partitions -------------------------------------------------------------
def partition(psi: int, nd: int, r: int) -> tuple[int, int]:
    b, e = _i64(), _i64()
    _partition(psi, nd, r, C.byref(b), C.byref(e))
    return b.value, e.value


chunk = partition


def shard_len(numel: Sequence[int], nd: int, r: int) -> int:
    n = np.ascontiguousarray(numel, dtype=np.int64)
    return int(_shard_len(len(n), _ptr(n), nd, r))


def bias_corrections(beta1: float, beta2: float, t: int) -> tuple[float, float]:
    a, b = _f32(), _f32()
    _bias(beta1, beta2, t, C.byref(a), C.byref(b))
    return np.float32(a.value), np.float32(b.value)


def inv_scale(loss_scale: float) -> np.float32:
    return np.float32(_inv_scale(loss_scale))


# ---- the step ---------------------------------------------------------------
def dp_step(grads: Sequence[np.ndarray], w, m, v, p16, loss_scale, hp: Hyper, t: int,
            decay=None):
    """Plain data-parallel definition. Returns (skipped, new_t). `decay`: optional
    per-element mask (nonzero = apply weight decay); None = every element."""
    gs = [_u16(g) for g in grads]
    n = w.size
    for g in gs:
        assert g.size == n
    tt = _i64(t)
    if decay is None:
        sk = _dp_step(n, len(gs), _ptrs(gs), _ptr(w), _ptr(m), _ptr(v), _ptr(_u16(p16)),
                      loss_scale, C.byref(hp), C.byref(tt))
    else:
        dm = np.ascontiguousarray(decay, dtype=np.uint8)
        assert dm.size == n
        sk = _dp_step_masked(n, len(gs), _ptrs(gs), _ptr(w), _ptr(m), _ptr(v), _ptr(_u16(p16)),
                             loss_scale, C.byref(hp), _ptr(dm), C.byref(tt))
    return bool(sk), tt.value


def decay_mask(numel: Sequence[int], no_decay: Sequence[bool]) -> np.ndarray:
    """Per-element mask of a tensor list: 0 on tensors excluded from weight decay."""
    return np.concatenate([np.full(int(n), 0 if nd else 1, np.uint8)
                           for n, nd in zip(numel, no_decay)])


def f32_from_bf16(h) -> np.ndarray:
    h = np.ascontiguousarray(h, dtype=np.uint16)
    out = np.empty(h.shape, np.float32)
    _f32_from_bf16_array(_ptr(h), _ptr(out), h.size)
    return out


def bf16_from_f32(x) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, np.uint16)
    _bf16_from_f32_array(_ptr(x), _ptr(out), x.size)
    return out


def bf16_from_f64_scalar(x: float) -> int:
    return int(_bf16_from_f64(float(x)))


def bf16_step(grads: Sequence[np.ndarray], w16, m, v, loss_scale, hp: Hyper, t: int, decay=None):
    """BF16 step without fp32 master weights; w16 (uint16 bfloat16 bits), m, v
    updated in place. Returns (skipped, new_t)."""
    gs = [np.ascontiguousarray(g, dtype=np.uint16) for g in grads]
    n = m.size
    assert w16.dtype == np.uint16 and w16.size == n and all(g.size == n for g in gs)
    dm = None if decay is None else np.ascontiguousarray(decay, dtype=np.uint8)
    tt = _i64(t)
    sk = _bf16_step(n, len(gs), _ptrs(gs), _ptr(w16), _ptr(m), _ptr(v), loss_scale, C.byref(hp),
                    None if dm is None else _ptr(dm), C.byref(tt))
    return bool(sk), tt.value


def zero12_step(psi, grads, w_sh, m_sh, v_sh, replicas, loss_scale, hp: Hyper, t: int):
    gs = [_u16(g) for g in grads]
    nd = len(gs)
    tt = _i64(t)
    sk = _z12_step(psi, nd, _ptrs(gs), _ptrs(w_sh), _ptrs(m_sh), _ptrs(v_sh),
                   _ptrs([_u16(r) for r in replicas]), loss_scale, C.byref(hp), C.byref(tt))
    return bool(sk), tt.value


def zero3_step(numel, grads, w_sh, m_sh, v_sh, p_sh, loss_scale, hp: Hyper, t: int):
    n = np.ascontiguousarray(numel, dtype=np.int64)
    gs = [_u16(g) for g in grads]
    tt = _i64(t)
    sk = _z3_step(len(n), _ptr(n), len(gs), _ptrs(gs), _ptrs(w_sh), _ptrs(m_sh), _ptrs(v_sh),
                  _ptrs([_u16(p) for p in p_sh]), loss_scale, C.byref(hp), C.byref(tt))
    return bool(sk), tt.value


def zero3_gather(numel, unit_of, nd, unit, p_sh) -> np.ndarray:
    n = np.ascontiguousarray(numel, dtype=np.int64)
    u = np.ascontiguousarray(unit_of, dtype=np.int32)
    total = int(n[u == unit].sum())
    out = np.empty(max(total, 1), np.uint16)
    got = _z3_gather(len(n), _ptr(n), _ptr(u), nd, unit, _ptrs([_u16(p) for p in p_sh]), _ptr(out))
    assert got == total
    return out[:total]


# ---- ledger -----------------------------------------------------------------
def ledger_formula(psi: float, nd: float) -> np.ndarray:
    out = (C.c_double * 4)()
    _formula(float(psi), float(nd), out)
    return np.array(out[:], dtype=np.float64)


def ledger_exact(psi: int, nd: int, numel: Sequence[int] | None = None) -> np.ndarray:
    out = (_i64 * 4)()
    if numel is None:
        _exact(psi, nd, 0, None, out)
    else:
        n = np.ascontiguousarray(numel, dtype=np.int64)
        _exact(psi, nd, len(n), _ptr(n), out)
    return np.array(out[:], dtype=np.int64)


def comm_elements(psi: int, nd: int) -> dict:
    out = (_i64 * 6)()
    _comm(psi, nd, out)
    keys = ["reduce_scatter", "all_gather", "dp", "stage1", "stage2", "stage3"]
    return dict(zip(keys, out[:]))


def scaler_update(scale: float, good: int, overflow: bool, growth: float, backoff: float,
                  interval: int) -> tuple[float, int]:
    sc, g = _f32(scale), _i32(good)
    _scaler(C.byref(sc), C.byref(g), int(overflow), growth, backoff, interval)
    return float(np.float32(sc.value)), g.value
