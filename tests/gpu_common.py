"""Shared helpers of the GPU parity tests: run a configuration through the C
ABI on the GPU and the same configuration through the oracle on the CPU, with
inputs from the seeded generator (host path for the oracle, and for small
cases the GPU gets the very same bits by copy).

Tolerances (the step's stated bar): master/m/v within max relative error
1e-6 (denominator max(|ref|, FLT_MIN)); fp16 parameters within 1 ulp; skip
decision and partition boundaries exact. The design is expected to be
bit-exact as well, and `compare_*` checks that too.
"""
from __future__ import annotations

import numpy as np
import torch

from oracle import zero_ref as Z
from zero_partitioned_mixed_02_b200 import _abi as A
from zero_partitioned_mixed_02_b200 import synth as S

FLT_MIN = np.float32(np.finfo(np.float32).tiny)
SENTINEL16 = 0x5A5A
GUARD = 64  # fp16 elements of guard band on each side of a parameter buffer


def dev_u16(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda()


def host_u16(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().numpy().view(np.uint16)


def host_f32(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().numpy().view(np.float32)


def compare_f32(got: np.ndarray, want: np.ndarray, what: str) -> None:
    got = np.asarray(got, np.float32)
    want = np.asarray(want, np.float32)
    assert got.shape == want.shape, (what, got.shape, want.shape)
    both_nan = np.isnan(got) & np.isnan(want)
    den = np.maximum(np.abs(want), FLT_MIN).astype(np.float64)
    rel = np.where(both_nan, 0.0, np.abs(got.astype(np.float64) - want) / den)
    worst = float(np.max(rel)) if rel.size else 0.0
    assert worst <= 1e-6, f"{what}: max relative error {worst:.3e} > 1e-6"
    same = (got.view(np.uint32) == want.view(np.uint32)) | both_nan
    assert same.all(), f"{what}: within tolerance but {int((~same).sum())} values not bit-identical"


def _ulp_index(h: np.ndarray) -> np.ndarray:
    """Monotone integer position of a binary16 value on the number line."""
    h = h.astype(np.int32)
    return np.where(h & 0x8000, -(h & 0x7FFF), h)


def compare_f16(got: np.ndarray, want: np.ndarray, what: str) -> None:
    got = np.asarray(got).view(np.uint16)
    want = np.asarray(want).view(np.uint16)
    assert got.shape == want.shape, (what, got.shape, want.shape)
    d = np.abs(_ulp_index(got) - _ulp_index(want))
    worst = int(d.max()) if d.size else 0
    assert worst <= 1, f"{what}: {worst} fp16 ulps apart"
    assert (got == want).all(), f"{what}: within 1 ulp but {int((got != want).sum())} differ"


class GuardedF16:
    """A device fp16 buffer with sentinel guard bands on both sides."""

    def __init__(self, n: int, fill_bits: np.ndarray | None = None):
        self.n = n
        host = np.full(n + 2 * GUARD, SENTINEL16, np.uint16)
        if fill_bits is not None:
            host[GUARD:GUARD + n] = fill_bits
        self.full = dev_u16(host)
        self.inner = self.full[GUARD:GUARD + n]

    def ptr(self) -> int:
        return self.inner.data_ptr()

    def bits(self) -> np.ndarray:
        return host_u16(self.inner)

    def guards_intact(self) -> bool:
        h = host_u16(self.full)
        return bool((h[:GUARD] == SENTINEL16).all() and (h[GUARD + self.n:] == SENTINEL16).all())


class GuardedWorkspace:
    def __init__(self, nbytes: int):
        self.g = 256
        self.full = torch.full((nbytes + 2 * self.g,), 0xA5, dtype=torch.uint8, device="cuda")
        self.nbytes = nbytes

    def ptr(self) -> int:
        return self.full.data_ptr() + self.g

    def guards_intact(self) -> bool:
        h = self.full.cpu().numpy()
        return bool((h[:self.g] == 0xA5).all() and (h[self.g + self.nbytes:] == 0xA5).all())

    def f32(self, byte_off: int, n: int) -> np.ndarray:
        b = self.g + byte_off
        return host_f32(self.full[b:b + 4 * n].view(torch.float32))

    def f32_at(self, byte_off: int, idx: np.ndarray) -> np.ndarray:
        b = self.g + byte_off
        n = int(idx.max()) + 1
        view = self.full[b:b + 4 * n].view(torch.float32)
        return host_f32(view[torch.from_numpy(idx).cuda()])

    def u16(self, byte_off: int, n: int) -> np.ndarray:
        b = self.g + byte_off
        return host_u16(self.full[b:b + 2 * n].view(torch.int16))


def state_offsets(h: int, ws: GuardedWorkspace) -> tuple[int, int, int, int]:
    w, m, v, t = A.zero_current_state(h)
    base = ws.ptr()
    # no master (bfloat16 without master weights): None
    return (None if w is None else w - base), m - base, v - base, t


def hyper(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.0) -> A.zero_hyper:
    return A.zero_hyper(lr, beta1, beta2, eps, weight_decay)
