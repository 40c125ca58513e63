"""Rank r of a real Nd-rank data-parallel job on the single-rank view.

Each process owns one GPU and one handle configured with rank_view = r and
view_outputs = nd: its step reads the Nd ranks' gradients of partition r
(peer-mapped pointers in a real job), updates partition r of master/m/v, and
writes the new fp16 partition into every rank's replica (again peer pointers):
the reduce-scatter and the all-gather of [P1] "The part that sounds too good:
communication" fused into the step. What is left to agree on is the overflow
decision: the step is skipped if any rank overflowed, so between the launch
and the commit the ranks reduce the handle's two flag words with MAX.

    skipped = rank_step(h, grads, loss_scale, hp, stream, group)

flag_words(h) is a zero-copy torch view of the two words (int32), usable
with torch.distributed.all_reduce on the NCCL backend.
"""
from __future__ import annotations

from typing import Sequence

import torch
import torch.distributed as dist

from . import _abi as A


class _DeviceWords:
    def __init__(self, ptr: int):
        self.__cuda_array_interface__ = {"shape": (2,), "typestr": "<i4", "data": (ptr, False),
                                         "version": 3, "strides": None}


def flag_words(h: int, device: torch.device | str | None = None) -> torch.Tensor:
    """The handle's overflow and kernel-error words as an int32[2] CUDA tensor
    sharing the handle's workspace memory."""
    return torch.as_tensor(_DeviceWords(A.zero_flag_words(h)), device=device or torch.device("cuda"))


def agree_overflow(words: torch.Tensor, group=None) -> torch.Tensor:
    """MAX-reduce the flag words across the group in place (the call id left
    by an overflowing rank wins; ids advance identically on every rank)."""
    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(words, op=dist.ReduceOp.MAX, group=group)
    return words


def rank_step(h: int, grads: Sequence[int], loss_scale: float, hp: A.zero_hyper,
              stream: torch.cuda.Stream, group=None) -> bool:
    """One step of this rank: enqueue, agree on overflow across ranks on the
    step's stream, commit. Returns True if the step was skipped."""
    A.zero_step_launch(h, grads, loss_scale, hp, stream.cuda_stream)
    with torch.cuda.stream(stream):
        agree_overflow(flag_words(h), group)
    return A.zero_step_commit(h, stream.cuda_stream) == A.ZERO_SKIPPED
