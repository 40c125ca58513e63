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

PeerBuffers exchanges descriptors of device buffers (include/zero_peer.h)
across the group and maps every rank's buffers into this process; PeerRank
is the whole per-rank job on top of it: this rank's gradient and parameter
buffers (stage 1/2) or gradient and shard-holding workspace (stage 3) shared
with the others, one handle, the step bracketed by device barriers, and on
stage 3 the layer gather from every rank's shard.
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
        agree_overflow_any(flag_words(h, stream.device), group)
    return A.zero_step_commit(h, stream.cuda_stream) == A.ZERO_SKIPPED


def _is_nccl(group=None) -> bool:
    return dist.get_backend(group) == "nccl"


def agree_overflow_any(words: torch.Tensor, group=None) -> torch.Tensor:
    """agree_overflow on any backend: NCCL reduces the device words in stream
    order; other backends (gloo) reduce a host copy, which waits for the
    current stream."""
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size(group) == 1:
        return words
    if _is_nccl(group) or words.device.type == "cpu":
        return agree_overflow(words, group)
    host = words.cpu()
    dist.all_reduce(host, op=dist.ReduceOp.MAX, group=group)
    words.copy_(host)
    return words


def device_barrier(stream: torch.cuda.Stream, group=None) -> None:
    """Order the GPU work of every rank: work enqueued on `stream` after this
    call starts only once every rank's work enqueued before its own call has
    finished. NCCL: a one-word all-reduce on the stream (no host wait); other
    backends: a stream synchronise and a host barrier."""
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size(group) == 1:
        return
    if _is_nccl(group):
        with torch.cuda.stream(stream):
            dist.all_reduce(torch.zeros(1, dtype=torch.int32, device=stream.device), group=group)
    else:
        stream.synchronize()
        dist.barrier(group=group)


class _ApiPeers:
    """The library's peer calls (include/zero_peer.h)."""
    export = staticmethod(A.zero_peer_export)
    open = staticmethod(A.zero_peer_open)
    close = staticmethod(A.zero_peer_close)


class PeerBuffers:
    """Every rank's counterpart of some local device buffers, addressable
    from this process. ptrs[k][j] is this process's address of rank k's j-th
    buffer (its own buffers are returned unchanged). Collective: every rank of
    the group constructs it with the same number of buffers, and close() is
    collective too (it waits until no rank can still use a mapping, then
    releases them)."""

    def __init__(self, buffers: Sequence[tuple[int, int]], group=None, api=_ApiPeers):
        """buffers: (device address, bytes) per local buffer."""
        self._api = api
        self._group = group
        mine = [api.export(int(p), int(n)) for p, n in buffers]
        world = dist.get_world_size(group)
        rows: list = [None] * world
        dist.all_gather_object(rows, mine, group=group)
        if any(len(r) != len(mine) for r in rows):
            raise ValueError("every rank must share the same number of buffers")
        self.descs = rows
        self.ptrs: list[list[int]] = []
        try:
            for row in rows:
                self.ptrs.append([])
                for d in row:
                    self.ptrs[-1].append(api.open(d))
        except Exception:
            self._release()
            raise

    def _release(self) -> None:
        for row, prow in zip(self.descs, self.ptrs):
            for d, p in zip(row, prow):
                self._api.close(d, p)
        self.ptrs = []

    def close(self, stream: torch.cuda.Stream | None = None) -> None:
        if stream is not None:
            stream.synchronize()
        dist.barrier(group=self._group)  # nobody is still reading or writing through a mapping
        self._release()
        dist.barrier(group=self._group)  # nobody frees a buffer another rank still maps


class PeerRank:
    """Rank r of a real Nd-rank job, one process per GPU (Nd = the group's
    size), on peer buffers.

    Stages 1 and 2: `grad` and `params` are this rank's full-length 16-bit
    gradient and parameter buffers (torch tensors of psi elements); the handle
    reads partition r of every rank's gradient and writes partition r of the
    new parameters into every rank's `params`; master_init holds partition r
    of the initial master weights.

    Stage 3: no parameter buffer (params=None): the handle reads chunk r of
    every tensor from every rank's gradient and keeps shard r of the fp16
    parameters in its workspace; gather(unit, out) assembles a layer unit from
    the Nd ranks' shards; master_init is the full flat master (every rank
    starts from the same weights) and `tensors` is required.

    step(): a device barrier (every rank's gradient is written), the step
    launch, the overflow agreement, the commit, and a second device barrier
    (every rank's new parameters, or shard, are complete)."""

    def __init__(self, grad: torch.Tensor, params: torch.Tensor | None, master_init: torch.Tensor,
                 stage: int = 2, variant: int = A.ZERO_VARIANT_FUSED_TMA,
                 precision: int = A.ZERO_PRECISION_FP16, tensors=None, group=None,
                 stream: torch.cuda.Stream | None = None):
        if stage not in (1, 2, 3):
            raise ValueError("stage 1, 2 or 3")
        psi = grad.numel()
        if grad.element_size() != 2:
            raise ValueError("grad: a 16-bit tensor")
        if stage <= 2:
            if params is None or params.numel() != psi or params.element_size() != 2:
                raise ValueError("params: a 16-bit tensor as long as grad")
        elif params is not None:
            raise ValueError("stage 3 keeps the parameters in shards: params=None")
        self.group = group
        self.stage = stage
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)
        self.stream = stream or torch.cuda.current_stream(grad.device)
        cfg_of = lambda r: A.Config(psi, self.world, stage, rank_view=r, variant=variant, tensors=tensors,
                                    precision=precision, view_outputs=self.world if stage <= 2 else 0)
        self.cfg = cfg_of(self.rank)
        L = A.zero_state_bytes(self.cfg)
        if stage <= 2:
            P = L.partition_len
            self.begin = min(self.rank * P, psi)
            self.end = min(self.begin + P, psi)
        else:
            self.begin, self.end = 0, psi
        if master_init.numel() != self.end - self.begin or master_init.dtype != torch.float32:
            raise ValueError(f"master_init: {self.end - self.begin} fp32 elements")
        self.workspace = torch.empty(L.workspace_bytes, dtype=torch.uint8, device=grad.device)
        second = params if stage <= 2 else self.workspace
        self.peers = PeerBuffers([(grad.data_ptr(), 2 * psi),
                                  (second.data_ptr(), second.numel() * second.element_size())], group)
        if stage <= 2:
            self.grad_ptrs = [row[0] + 2 * self.begin for row in self.peers.ptrs]
            outs = [row[1] for row in self.peers.ptrs]
            self.shard_ptrs = None
        else:
            self.grad_ptrs = [row[0] for row in self.peers.ptrs]
            outs = None
            # rank k's shard sits at its own layout's offset in its workspace
            self.shard_ptrs = [row[1] + A.zero_state_bytes(cfg_of(k)).off_shard16
                               for k, row in enumerate(self.peers.ptrs)]
        self.h = None
        try:
            self.h = A.zero_init(self.cfg, self.workspace.data_ptr(), L.workspace_bytes,
                                 master_init.data_ptr(), outs, self.stream.cuda_stream)
        finally:
            # every rank's initial parameters are in place (or every rank
            # learns here that one of them failed: the barrier ends)
            device_barrier(self.stream, group)
        self._grads = grad
        self._params = params

    def step(self, loss_scale: float, hp: A.zero_hyper) -> bool:
        device_barrier(self.stream, self.group)
        skipped = rank_step(self.h, self.grad_ptrs, loss_scale, hp, self.stream, self.group)
        device_barrier(self.stream, self.group)
        return skipped

    def unit_range(self, unit: int) -> tuple[int, int]:
        """Flat offset and length of a layer unit (stage 3)."""
        return A.zero_unit_range(self.cfg, unit)

    def gather(self, unit: int, out: torch.Tensor) -> torch.Tensor:
        """Stage 3: layer unit `unit` from the Nd ranks' shards into `out` (a
        16-bit tensor of the unit's length), on this rank's stream. Local: the
        shards it reads were completed by the step's closing barrier."""
        if self.stage != 3:
            raise ValueError("gather: stage 3 only")
        _, n = self.unit_range(unit)
        if out.numel() < n or out.element_size() != 2:
            raise ValueError(f"out: at least {n} 16-bit elements")
        A.zero_gather_layer_ranks(self.h, unit, self.shard_ptrs, out.data_ptr(), self.stream.cuda_stream)
        return out

    def state(self) -> tuple[int, int, int, int]:
        """Device addresses of this rank's master, m, v and t."""
        return A.zero_current_state(self.h)

    def close(self) -> None:
        self.stream.synchronize()
        if self.h is not None:
            A.zero_destroy(self.h)
            self.h = None
        self.peers.close(self.stream)
