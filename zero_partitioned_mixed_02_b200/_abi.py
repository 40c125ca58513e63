"""ctypes binding of libzero's C ABI (include/zero.h), same names, argument
marshalling only: every step of the optimizer runs in libzero's kernels.

Device pointers are passed as Python ints (``tensor.data_ptr()``), streams as
``torch.cuda.Stream.cuda_stream`` ints. Errors raise ``ZeroError``; the
informational ZERO_SKIPPED is returned, not raised.
"""
from __future__ import annotations

import ctypes as C
import os
from typing import Sequence

PKG = os.path.dirname(os.path.abspath(__file__))
# ZERO_LIBZERO selects another build of the library (the bounds-checked
# libzero_bounds.so); it must exist like the default one
LIB_PATH = os.environ.get("ZERO_LIBZERO") or os.path.join(PKG, "libzero.so")

ZERO_OK = 0
ZERO_SKIPPED = 1
ZERO_ERR_ARG = -1
ZERO_ERR_ALIGN = -2
ZERO_ERR_STAGE = -3
ZERO_ERR_WORKSPACE = -4
ZERO_ERR_CUDA = -5
ZERO_ERR_INTERNAL = -6
ZERO_ERR_PARTIAL = -7

ZERO_TENSOR_NO_DECAY = 1
ZERO_PRECISION_FP16 = 0
ZERO_PRECISION_BF16 = 1

ZERO_VARIANT_FUSED = 0
ZERO_VARIANT_TWO_PASS = 1
ZERO_VARIANT_FUSED_TMA = 2
ZERO_VARIANT_TWO_PASS_TMA = 3
ZERO_MAX_ND = 1024


class ZeroError(RuntimeError):
    def __init__(self, code: int, where: str, cuda: int = 0):
        msg = f"{where}: {error_string(code)} ({code})"
        if cuda:
            msg += f", cudaError {cuda}"
        super().__init__(msg)
        self.code = code


class zero_tensor(C.Structure):
    _fields_ = [("numel", C.c_int64), ("unit", C.c_int32), ("flags", C.c_int32)]


class zero_config(C.Structure):
    _fields_ = [("psi", C.c_int64), ("nd", C.c_int32), ("stage", C.c_int32),
                ("rank_view", C.c_int32), ("variant", C.c_int32), ("n_tensors", C.c_int32),
                ("precision", C.c_int32), ("tensors", C.POINTER(zero_tensor)),
                ("view_outputs", C.c_int32), ("reserved", C.c_int32)]


class zero_hyper(C.Structure):
    _fields_ = [("lr", C.c_float), ("beta1", C.c_float), ("beta2", C.c_float),
                ("eps", C.c_float), ("weight_decay", C.c_float)]


class zero_scaler(C.Structure):
    _fields_ = [("init_scale", C.c_float), ("growth_factor", C.c_float),
                ("backoff_factor", C.c_float), ("growth_interval", C.c_int32)]


class zero_async_state(C.Structure):
    _fields_ = [("t", C.c_int64), ("skipped", C.c_int64), ("loss_scale", C.c_float),
                ("good_steps", C.c_int32)]


class zero_ledger(C.Structure):
    _fields_ = [("formula_bytes", C.c_double * 4), ("exact_bytes", C.c_int64 * 4),
                ("comm_elements", C.c_int64 * 6), ("allreduce_buffer_bytes", C.c_int64),
                ("transient_bytes", C.c_int64), ("peak_stage3_bytes", C.c_int64),
                ("workspace_bytes", C.c_int64), ("partition_len", C.c_int64),
                ("state_elems", C.c_int64), ("grad_len", C.c_int64),
                ("off_master", C.c_int64 * 2), ("off_m", C.c_int64 * 2), ("off_v", C.c_int64 * 2),
                ("off_shard16", C.c_int64), ("off_reduced", C.c_int64),
                ("n_units", C.c_int32), ("n_out", C.c_int32)]


class zero_offload_ledger(C.Structure):
    _fields_ = [("state_elems", C.c_int64), ("host_state_bytes", C.c_int64),
                ("host_staging_bytes", C.c_int64), ("device_bytes", C.c_int64),
                ("chunk_elems", C.c_int64), ("n_chunks", C.c_int64),
                ("d2h_bytes_per_step", C.c_int64), ("h2d_bytes_per_step", C.c_int64),
                ("device_state_bytes", C.c_int64), ("n_out", C.c_int32), ("reserved", C.c_int32)]


ZERO_OFFLOAD_SLOTS = 3
ZERO_OFFLOAD_DEFAULT_CHUNK = 1 << 22


class zero_gather_run(C.Structure):
    _fields_ = [("src_begin", C.c_int64), ("out_begin", C.c_int64), ("len", C.c_int64),
                ("src_rank", C.c_int32), ("reserved", C.c_int32)]


class zero_peer_desc(C.Structure):
    _fields_ = [("magic", C.c_uint32), ("device", C.c_int32), ("process", C.c_uint64),
                ("offset", C.c_uint64), ("bytes", C.c_uint64), ("address", C.c_uint64),
                ("ipc", C.c_ubyte * 64)]


ZERO_PEER_MAGIC = 0x5A505231
ZERO_PEER_DESC_BYTES = 104

_lib = None


def lib():
    """Load libzero.so. Raises if the extension is not built: there is no
    fallback path."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libzero.so not built at {LIB_PATH}; "
                               "run python -m zero_partitioned_mixed_02_b200.build")
        L = C.CDLL(LIB_PATH)
        P = C.c_void_p
        sig = {
            "zero_state_bytes": (C.c_int, [C.POINTER(zero_config), C.POINTER(zero_ledger)]),
            "zero_rank_shard": (C.c_int, [C.POINTER(zero_config), C.c_int32,
                                          C.POINTER(C.c_int64), C.POINTER(C.c_int64)]),
            "zero_unit_range": (C.c_int, [C.POINTER(zero_config), C.c_int32,
                                          C.POINTER(C.c_int64), C.POINTER(C.c_int64)]),
            "zero_init": (C.c_int, [C.POINTER(zero_config), P, C.c_size_t, P, C.POINTER(P), P,
                                    C.POINTER(P)]),
            "zero_step": (C.c_int, [P, C.POINTER(P), C.c_float, C.POINTER(zero_hyper), P,
                                    C.POINTER(C.c_int)]),
            "zero_step_launch": (C.c_int, [P, C.POINTER(P), C.c_float, C.POINTER(zero_hyper), P]),
            "zero_step_commit": (C.c_int, [P, P, C.POINTER(C.c_int)]),
            "zero_gather_layer": (C.c_int, [P, C.c_int32, P, P]),
            "zero_gather_layer_ranks": (C.c_int, [P, C.c_int32, C.POINTER(P), P, P]),
            "zero_gather_plan": (C.c_int, [C.POINTER(zero_config), C.c_int32, C.POINTER(zero_gather_run),
                                           C.c_int64, C.POINTER(C.c_int64)]),
            "zero_async_begin": (C.c_int, [P, C.POINTER(P), C.POINTER(zero_scaler), C.c_float,
                                           C.c_float, P]),
            "zero_step_async": (C.c_int, [P, C.POINTER(zero_hyper), P]),
            "zero_async_end": (C.c_int, [P, P, C.POINTER(zero_async_state)]),
            "zero_current_state": (C.c_int, [P, C.POINTER(P), C.POINTER(P), C.POINTER(P),
                                             C.POINTER(C.c_int64)]),
            "zero_stream_copy": (C.c_int, [P, P, C.c_size_t, P]),
            "zero_set_state": (C.c_int, [P, P, P, P, C.c_int64, P]),
            "zero_step_static": (C.c_int, [C.c_int64, C.c_int32, C.POINTER(P), P, P, P, C.POINTER(P),
                                           C.c_float, C.POINTER(zero_hyper),
                                           C.POINTER(C.c_int64), P, C.POINTER(C.c_int)]),
            "zero_last_cuda_error": (C.c_int, [P]),
            "zero_uses_tma": (C.c_int, [P]),
            "zero_flag_words": (C.c_int, [P, C.POINTER(P)]),
            "zero_test_hold_tile": (C.c_int, [P, C.c_int64, C.c_uint32]),
            "zero_test_hold_update_tile": (C.c_int, [P, C.c_int64, C.c_uint32]),
            "zero_error_string": (C.c_char_p, [C.c_int]),
            "zero_destroy": (None, [P]),
            "zero_offload_bytes": (C.c_int, [C.POINTER(zero_config), C.c_int64,
                                             C.POINTER(zero_offload_ledger)]),
            "zero_offload_init": (C.c_int, [C.POINTER(zero_config), C.c_int64, P, C.c_size_t, P,
                                            C.c_size_t, P, P, C.POINTER(P), C.c_int, P,
                                            C.POINTER(P)]),
            "zero_offload_step": (C.c_int, [P, C.POINTER(P), C.c_float, C.POINTER(zero_hyper), P]),
            "zero_offload_state": (C.c_int, [P, C.POINTER(P), C.POINTER(P), C.POINTER(P),
                                             C.POINTER(C.c_int64)]),
            "zero_offload_set_state": (C.c_int, [P, P, P, P, C.c_int64, P]),
            "zero_offload_gather_layer": (C.c_int, [P, C.c_int32, P, P]),
            "zero_offload_host_update": (C.c_int, [P, P, P, P, P, C.c_int64, C.POINTER(zero_hyper),
                                                   C.c_int64, C.c_int, C.c_int]),
            "zero_offload_destroy": (None, [P]),
            "zero_peer_export": (C.c_int, [P, C.c_size_t, C.POINTER(zero_peer_desc)]),
            "zero_peer_open": (C.c_int, [C.POINTER(zero_peer_desc), C.POINTER(P)]),
            "zero_peer_close": (C.c_int, [C.POINTER(zero_peer_desc), P]),
            "zero_peer_open_count": (C.c_int, []),
            "zero_peer_last_cuda_error": (C.c_int, []),
        }
        for name, (res, args) in sig.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def error_string(code: int) -> str:
    return lib().zero_error_string(code).decode()


class Config:
    """zero_config plus the tensor array it points to (kept alive together)."""

    def __init__(self, psi: int, nd: int, stage: int, rank_view: int = -1,
                 variant: int = ZERO_VARIANT_FUSED,
                 tensors: Sequence[tuple[int, ...]] | None = None,
                 precision: int = ZERO_PRECISION_FP16, view_outputs: int = 0):
        """tensors: (numel, unit) or (numel, unit, flags) per tensor, flat order;
        flags = ZERO_TENSOR_NO_DECAY excludes the tensor from weight decay."""
        self._tensors = None
        n = 0
        ptr = None
        if tensors:
            n = len(tensors)
            self._tensors = (zero_tensor * n)(*[
                zero_tensor(int(t[0]), int(t[1]), int(t[2]) if len(t) > 2 else 0) for t in tensors])
            ptr = C.cast(self._tensors, C.POINTER(zero_tensor))
        self.c = zero_config(int(psi), int(nd), int(stage), int(rank_view), int(variant), n,
                             int(precision), ptr, int(view_outputs), 0)

    def byref(self):
        return C.byref(self.c)


def _check(rc: int, where: str, h=None) -> int:
    if rc < 0:
        cuda = lib().zero_last_cuda_error(h) if h else 0
        raise ZeroError(rc, where, cuda)
    return rc


def zero_state_bytes(cfg: Config) -> zero_ledger:
    out = zero_ledger()
    _check(lib().zero_state_bytes(cfg.byref(), C.byref(out)), "zero_state_bytes")
    return out


def zero_rank_shard(cfg: Config, rank: int) -> tuple[int, int]:
    b, n = C.c_int64(), C.c_int64()
    _check(lib().zero_rank_shard(cfg.byref(), rank, C.byref(b), C.byref(n)), "zero_rank_shard")
    return b.value, n.value


def zero_unit_range(cfg: Config, unit: int) -> tuple[int, int]:
    b, n = C.c_int64(), C.c_int64()
    _check(lib().zero_unit_range(cfg.byref(), unit, C.byref(b), C.byref(n)), "zero_unit_range")
    return b.value, n.value


def _ptr_array(ptrs: Sequence[int] | None):
    if ptrs is None:
        return None
    return (C.c_void_p * max(len(ptrs), 1))(*[int(p) for p in ptrs])


def zero_init(cfg: Config, workspace: int, workspace_bytes: int, master_init: int,
              param_bufs: Sequence[int] | None, stream: int) -> int:
    h = C.c_void_p()
    arr = _ptr_array(param_bufs)
    _check(lib().zero_init(cfg.byref(), workspace, workspace_bytes, master_init, arr, stream,
                           C.byref(h)), "zero_init")
    return h.value


def zero_step(h: int, grads: Sequence[int], loss_scale: float, hp: zero_hyper, stream: int) -> int:
    arr = _ptr_array(grads)
    sk = C.c_int(0)
    return _check(lib().zero_step(h, arr, float(loss_scale), C.byref(hp), stream, C.byref(sk)),
                  "zero_step", h)


def zero_step_launch(h: int, grads: Sequence[int], loss_scale: float, hp: zero_hyper,
                     stream: int) -> None:
    arr = _ptr_array(grads)
    _check(lib().zero_step_launch(h, arr, float(loss_scale), C.byref(hp), stream),
           "zero_step_launch", h)


def zero_step_commit(h: int, stream: int) -> int:
    sk = C.c_int(0)
    return _check(lib().zero_step_commit(h, stream, C.byref(sk)), "zero_step_commit", h)


def zero_async_begin(h: int, grads: Sequence[int], sc: zero_scaler, beta1: float, beta2: float,
                     stream: int) -> None:
    _check(lib().zero_async_begin(h, _ptr_array(grads), C.byref(sc), beta1, beta2, stream),
           "zero_async_begin", h)


def zero_step_async(h: int, hp: zero_hyper, stream: int) -> None:
    _check(lib().zero_step_async(h, C.byref(hp), stream), "zero_step_async", h)


def zero_async_end(h: int, stream: int) -> zero_async_state:
    out = zero_async_state()
    _check(lib().zero_async_end(h, stream, C.byref(out)), "zero_async_end", h)
    return out


def zero_gather_layer(h: int, unit: int, out: int, stream: int) -> None:
    _check(lib().zero_gather_layer(h, unit, out, stream), "zero_gather_layer", h)


def zero_gather_layer_ranks(h: int, unit: int, shards: Sequence[int], out: int, stream: int) -> None:
    """Stage-3 rank of a real job: gather a layer unit from the Nd ranks'
    fp16 shards (shards[k]: rank k's shard, peer-mapped for other ranks)."""
    _check(lib().zero_gather_layer_ranks(h, unit, _ptr_array(shards), out, stream), "zero_gather_layer_ranks", h)


def zero_gather_plan(cfg: Config, unit: int) -> list[tuple[int, int, int, int]]:
    """The copies of a stage-3 layer gather: (src_rank, src_begin, out_begin, len)."""
    n = C.c_int64()
    _check(lib().zero_gather_plan(cfg.byref(), unit, None, 0, C.byref(n)), "zero_gather_plan")
    runs = (zero_gather_run * max(n.value, 1))()
    _check(lib().zero_gather_plan(cfg.byref(), unit, runs, n.value, C.byref(n)), "zero_gather_plan")
    return [(r.src_rank, r.src_begin, r.out_begin, r.len) for r in runs[:n.value]]


def zero_current_state(h: int) -> tuple[int, int, int, int]:
    w, m, v = C.c_void_p(), C.c_void_p(), C.c_void_p()
    t = C.c_int64()
    _check(lib().zero_current_state(h, C.byref(w), C.byref(m), C.byref(v), C.byref(t)),
           "zero_current_state")
    return w.value, m.value, v.value, t.value


def zero_set_state(h: int, master: int, m: int, v: int, t: int, stream: int) -> None:
    _check(lib().zero_set_state(h, master, m, v, t, stream), "zero_set_state", h)


def zero_stream_copy(dst: int, src: int, nbytes: int, stream: int) -> None:
    _check(lib().zero_stream_copy(dst, src, nbytes, stream), "zero_stream_copy")


ZERO_STATIC_MAX_PSI = 1048576
ZERO_STATIC_MAX_ND = 64


def zero_step_static(psi: int, grads: Sequence[int], master: int, m: int, v: int,
                     replicas: Sequence[int], loss_scale: float, hp: zero_hyper, t: int,
                     stream: int) -> tuple[int, int]:
    """Allocation-free two-pass step (scratch inside the library).
    Returns (return code, new t)."""
    tt = C.c_int64(t)
    sk = C.c_int(0)
    rc = _check(lib().zero_step_static(psi, len(grads), _ptr_array(grads), master, m, v,
                                       _ptr_array(replicas), float(loss_scale), C.byref(hp),
                                       C.byref(tt), stream, C.byref(sk)), "zero_step_static")
    return rc, tt.value


def zero_test_hold_tile(h: int, tile: int, wait_rounds: int) -> None:
    _check(lib().zero_test_hold_tile(h, tile, wait_rounds), "zero_test_hold_tile")


def zero_test_hold_update_tile(h: int, tile: int, wait_rounds: int) -> None:
    _check(lib().zero_test_hold_update_tile(h, tile, wait_rounds), "zero_test_hold_update_tile")


def zero_flag_words(h: int) -> int:
    """Device address of the handle's overflow and kernel-error words (two uint32)."""
    p = C.c_void_p()
    _check(lib().zero_flag_words(h, C.byref(p)), "zero_flag_words")
    return p.value


def zero_uses_tma(h: int) -> bool:
    return _check(lib().zero_uses_tma(h), "zero_uses_tma") == 1


def zero_destroy(h: int) -> None:
    lib().zero_destroy(h)


# ---- offloaded step (include/zero_offload.h) ----

def zero_offload_bytes(cfg: Config, chunk_elems: int = 0) -> zero_offload_ledger:
    out = zero_offload_ledger()
    _check(lib().zero_offload_bytes(cfg.byref(), int(chunk_elems), C.byref(out)), "zero_offload_bytes")
    return out


def zero_offload_init(cfg: Config, chunk_elems: int, device_ws: int, device_bytes: int,
                      host_staging: int, staging_bytes: int, host_state: int, master_init: int,
                      param_bufs: Sequence[int], n_threads: int, stream: int) -> int:
    h = C.c_void_p()
    _check(lib().zero_offload_init(cfg.byref(), int(chunk_elems), device_ws, device_bytes, host_staging,
                                   staging_bytes, host_state, master_init, _ptr_array(param_bufs),
                                   int(n_threads), stream, C.byref(h)), "zero_offload_init")
    return h.value


def zero_offload_step(h: int, grads: Sequence[int], loss_scale: float, hp: zero_hyper,
                      stream: int) -> int:
    return _check(lib().zero_offload_step(h, _ptr_array(grads), float(loss_scale), C.byref(hp), stream),
                  "zero_offload_step")


def zero_offload_state(h: int) -> tuple[int, int, int, int]:
    w, m, v = C.c_void_p(), C.c_void_p(), C.c_void_p()
    t = C.c_int64()
    _check(lib().zero_offload_state(h, C.byref(w), C.byref(m), C.byref(v), C.byref(t)),
           "zero_offload_state")
    return w.value, m.value, v.value, t.value


def zero_offload_gather_layer(h: int, unit: int, out: int, stream: int) -> None:
    _check(lib().zero_offload_gather_layer(h, unit, out, stream), "zero_offload_gather_layer")


def zero_offload_set_state(h: int, master: int, m: int, v: int, t: int, stream: int) -> None:
    _check(lib().zero_offload_set_state(h, master, m, v, int(t), stream), "zero_offload_set_state")


def zero_offload_host_update(g: int, w: int, m: int, v: int, p16: int, n: int, hp: zero_hyper, t: int,
                             decay: bool, path: int = 0) -> None:
    _check(lib().zero_offload_host_update(g, w, m, v, p16, int(n), C.byref(hp), int(t), int(bool(decay)),
                                          int(path)), "zero_offload_host_update")


def zero_offload_destroy(h: int) -> None:
    lib().zero_offload_destroy(h)


# ---- peer buffers (include/zero_peer.h) ----

def _peer_check(rc: int, where: str) -> int:
    if rc < 0:
        raise ZeroError(rc, where, lib().zero_peer_last_cuda_error())
    return rc


def _desc(desc: bytes) -> zero_peer_desc:
    if len(desc) != C.sizeof(zero_peer_desc):
        raise ZeroError(ZERO_ERR_ARG, "peer descriptor length")
    return zero_peer_desc.from_buffer_copy(desc)


def zero_peer_export(dev_ptr: int, nbytes: int) -> bytes:
    """Descriptor (104 bytes) of the device buffer [dev_ptr, dev_ptr + nbytes)."""
    d = zero_peer_desc()
    _peer_check(lib().zero_peer_export(dev_ptr, int(nbytes), C.byref(d)), "zero_peer_export")
    return bytes(d)


def zero_peer_open(desc: bytes) -> int:
    """This process's address of the buffer a descriptor names."""
    p = C.c_void_p()
    _peer_check(lib().zero_peer_open(C.byref(_desc(desc)), C.byref(p)), "zero_peer_open")
    return p.value


def zero_peer_close(desc: bytes, dev_ptr: int) -> None:
    _peer_check(lib().zero_peer_close(C.byref(_desc(desc)), dev_ptr), "zero_peer_close")


def zero_peer_open_count() -> int:
    return lib().zero_peer_open_count()
