"""Stage-3 layer gathers with prefetch: a double-buffered transient and a side
stream ([P3] "Partitioned parameters still have to participate in
computation": prefetch can hide transfer time while consuming additional
memory; [P3] "Check your understanding": the gathered layer is a peak that
does not divide by Nd).

    pf = LayerPrefetcher(opt.h, opt.ledger, stream)
    for unit, weights in pf.walk(forward_then_backward_order):
        ...  # use `weights` (int16 view of the fp16 bits) on `stream`

While the caller works on unit i on its stream, unit i+1 is gathered into the
other buffer on the side stream. Ordering is by CUDA events only (the host
never waits): a gather into a buffer waits for the caller's use of the unit
that buffer held before, and the caller's stream waits for the gather of the
unit it is handed. Peak transient memory is two units instead of one.
"""
from __future__ import annotations

from typing import Iterable, Iterator

import torch

from . import _abi as A


class LayerPrefetcher:
    def __init__(self, handle: int, ledger, stream: torch.cuda.Stream | None = None,
                 device: torch.device | str = "cuda", priority: int = 0):
        """priority: of the side stream (lower is higher, see
        torch.cuda.Stream); a high priority lets the gather's CTAs take SMs as
        the caller's kernel frees them."""
        if ledger.n_units <= 0:
            raise ValueError("layer gathers need a stage-3 handle")
        self.h = handle
        self.stream = stream or torch.cuda.current_stream(device)
        self.side = torch.cuda.Stream(device=self.stream.device, priority=priority)
        n = max(ledger.transient_bytes // 2, 1)
        self.buffers = [torch.empty(n, dtype=torch.int16, device=self.stream.device) for _ in range(2)]
        self.peak_bytes = 2 * ledger.transient_bytes

    def _gather(self, unit: int, b: int, released: list) -> torch.cuda.Event:
        if released[b] is not None:
            self.side.wait_event(released[b])
        A.zero_gather_layer(self.h, unit, self.buffers[b].data_ptr(), self.side.cuda_stream)
        done = torch.cuda.Event()
        done.record(self.side)
        return done

    def walk(self, order: Iterable[int], unit_numel=None) -> Iterator[tuple[int, torch.Tensor]]:
        """Yield (unit, gathered weights) in `order`; the weights tensor is a
        view valid until the next item is requested. `unit_numel(u)` gives the
        element count to expose (default: the whole buffer)."""
        order = list(order)
        if not order:
            return
        released = [None, None]
        # the side stream must not start before work already queued on the
        # caller's stream (the step that wrote the shards)
        start = torch.cuda.Event()
        start.record(self.stream)
        self.side.wait_event(start)
        gathered = {0: self._gather(order[0], 0, released)}
        for i, unit in enumerate(order):
            b = i % 2
            if i + 1 < len(order):
                gathered[i + 1] = self._gather(order[i + 1], 1 - b, released)
            self.stream.wait_event(gathered.pop(i))
            w = self.buffers[b]
            if unit_numel is not None:
                w = w[: unit_numel(unit)]
            yield unit, w
            ev = torch.cuda.Event()
            ev.record(self.stream)
            released[b] = ev
        # later work on the side stream (none) and the caller's stream are ordered
        tail = torch.cuda.Event()
        tail.record(self.side)
        self.stream.wait_event(tail)
