"""User-facing object over the C ABI: PyTorch allocates the device memory and
supplies the stream; libzero does all the work.

    opt = ZeroAdam(psi, nd, stage, master_init, param_bufs, tensors=..., variant=...)
    skipped = opt.step(grads, loss_scale, lr=..., betas=..., eps=..., weight_decay=...)
    opt.gather_layer(unit, out)          # stage 3
    w, m, v = opt.state()                # live fp32 state (views of the workspace)
    sd = opt.state_dict(); opt.load_state_dict(sd)     # checkpoint / resume
    opt.begin_async(grads, scaler); opt.step_async(...); opt.end_async()

    off = ZeroOffloadAdam(psi, nd, stage, master_init_host, param_bufs)   # host fp32 state
    skipped = off.step(grads, loss_scale, lr=...)
"""
from __future__ import annotations

from typing import Sequence

import torch

from . import _abi as A


class ZeroPartialUpdateError(A.ZeroError):
    """The in-place update pass of a two-pass TMA step gave up a bounded wait
    part of the way (ZERO_ERR_PARTIAL): some elements of the master (without
    one, the 16-bit weights), m, v and the parameters hold the new step's
    values, the others the previous step's, and t did not advance. Nothing can
    be rolled back inside the library; restore the state saved before the step
    with load_state_dict (which rewrites the parameters as well) and run the
    step again."""


class ZeroAdam:
    def __init__(self, psi: int, nd: int, stage: int, master_init: torch.Tensor,
                 param_bufs: Sequence[torch.Tensor] | None = None, *, rank_view: int = -1,
                 variant: int = A.ZERO_VARIANT_FUSED_TMA,
                 tensors: Sequence[tuple[int, ...]] | None = None,
                 stream: torch.cuda.Stream | None = None,
                 precision: int = A.ZERO_PRECISION_FP16):
        """precision = ZERO_PRECISION_BF16: bfloat16 gradients and parameters
        without fp32 master weights. The fused variants then roll back from the
        last replica, so they exist for stage 1/2 with all Nd >= 2 ranks; for
        anything else a fused variant is replaced by ZERO_VARIANT_TWO_PASS_TMA."""
        if (precision == A.ZERO_PRECISION_BF16 and variant in (A.ZERO_VARIANT_FUSED, A.ZERO_VARIANT_FUSED_TMA)
                and not (stage <= 2 and rank_view < 0 and nd >= 2)):
            variant = A.ZERO_VARIANT_TWO_PASS_TMA
        self.cfg = A.Config(psi, nd, stage, rank_view=rank_view, variant=variant, tensors=tensors,
                            precision=precision)
        self.ledger = A.zero_state_bytes(self.cfg)
        dev = master_init.device
        if dev.type != "cuda":
            raise ValueError("master_init must be a CUDA tensor")
        if master_init.dtype != torch.float32 or not master_init.is_contiguous():
            raise ValueError("master_init must be contiguous float32")
        self.stream = stream or torch.cuda.current_stream(dev)
        self.workspace = torch.empty(self.ledger.workspace_bytes, dtype=torch.uint8, device=dev)
        self.param_bufs = list(param_bufs) if param_bufs is not None else None
        ptrs = [p.data_ptr() for p in self.param_bufs] if self.param_bufs is not None else None
        self.h = A.zero_init(self.cfg, self.workspace.data_ptr(), self.ledger.workspace_bytes,
                             master_init.data_ptr(), ptrs, self.stream.cuda_stream)
        self.nd = nd

    def step(self, grads: Sequence[torch.Tensor] | Sequence[int], loss_scale: float, *, lr=1e-3,
             betas=(0.9, 0.999), eps=1e-8, weight_decay=0.0) -> bool:
        ptrs = [g if isinstance(g, int) else g.data_ptr() for g in grads]
        if len(ptrs) != self.nd:
            raise ValueError(f"expected {self.nd} gradient buffers, got {len(ptrs)}")
        hp = A.zero_hyper(lr, betas[0], betas[1], eps, weight_decay)
        try:
            rc = A.zero_step(self.h, ptrs, loss_scale, hp, self.stream.cuda_stream)
        except A.ZeroError as e:
            if e.code == A.ZERO_ERR_PARTIAL:
                raise ZeroPartialUpdateError(e.code, "ZeroAdam.step: the state is partly updated; restore a "
                                                     "saved state_dict with load_state_dict") from e
            raise
        return rc == A.ZERO_SKIPPED

    def gather_layer(self, unit: int, out: torch.Tensor) -> None:
        A.zero_gather_layer(self.h, unit, out.data_ptr(), self.stream.cuda_stream)

    def unit_range(self, unit: int) -> tuple[int, int]:
        return A.zero_unit_range(self.cfg, unit)

    def rank_shard(self, rank: int) -> tuple[int, int]:
        return A.zero_rank_shard(self.cfg, rank)

    @property
    def t(self) -> int:
        return A.zero_current_state(self.h)[3]

    def _view_f32(self, ptr: int | None) -> torch.Tensor | None:
        if ptr is None:
            return None  # no master (bfloat16 without master weights)
        off = ptr - self.workspace.data_ptr()
        n = self.ledger.state_elems
        return self.workspace[off: off + 4 * n].view(torch.float32)

    def state(self) -> tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
        w, m, v, _ = A.zero_current_state(self.h)
        return self._view_f32(w), self._view_f32(m), self._view_f32(v)

    def shard16(self) -> torch.Tensor:
        """Stage 3: the fp16 parameter shards (state order: every rank's when
        emulating all ranks, this rank's alone for a rank view), as int16 bits."""
        off = self.ledger.off_shard16
        if off < 0:
            raise ValueError("only stage 3 keeps fp16 shards")
        n = self.ledger.state_elems
        return self.workspace[off: off + 2 * n].view(torch.int16)

    def weights16(self) -> torch.Tensor:
        """The 16-bit parameters of the state's elements, in state order, as
        int16 bits: the shard (stage 3), this rank's partition of its
        parameter buffer (a rank view), or the first replica (stage 1/2)."""
        if self.ledger.off_shard16 >= 0:
            return self.shard16()
        if self.cfg.c.rank_view >= 0:
            b = min(self.cfg.c.rank_view * self.ledger.partition_len, self.cfg.c.psi)
            return self.param_bufs[0].view(torch.int16)[b: b + self.ledger.state_elems]
        return self.param_bufs[0].view(torch.int16)[: self.ledger.state_elems]

    def state_dict(self) -> dict:
        """Copies of master (None without one), m, v (state order) and the step
        count. Without a master (bfloat16) it also holds "weights": the
        bfloat16 parameters widened to float32 (exact), which load_state_dict
        writes back; a step that stopped part of the way
        (ZeroPartialUpdateError) may have changed them."""
        w, m, v = self.state()
        sd = {"master": None if w is None else w.clone(), "m": m.clone(), "v": v.clone(), "t": self.t}
        if w is None:
            sd["weights"] = self.weights16().view(torch.bfloat16).to(torch.float32)
        return sd

    def load_state_dict(self, sd: dict) -> None:
        """Restore master/m/v and t, and rewrite the 16-bit parameters from
        the master (without a master: from sd["weights"] if present, else
        they are left as they are)."""
        w = sd["master"] if sd["master"] is not None else sd.get("weights")
        tensors = [x for x in (w, sd["m"], sd["v"]) if x is not None]
        for x in tensors:
            if x.dtype != torch.float32 or not x.is_cuda or x.numel() != self.ledger.state_elems:
                raise ValueError("state tensors must be CUDA float32 of ledger.state_elems elements")
        w = None if w is None else w.contiguous()
        m, v = sd["m"].contiguous(), sd["v"].contiguous()
        A.zero_set_state(self.h, 0 if w is None else w.data_ptr(), m.data_ptr(), v.data_ptr(), int(sd["t"]),
                         self.stream.cuda_stream)

    def begin_async(self, grads: Sequence[torch.Tensor], init_scale: float = 65536.0,
                    growth_factor: float = 2.0, backoff_factor: float = 0.5,
                    growth_interval: int = 2000, betas=(0.9, 0.999)) -> None:
        """Open an asynchronous run on fixed gradient buffers (refill them
        between steps): steps then run without host synchronisation, with a
        dynamic loss scale kept on the device."""
        sc = A.zero_scaler(init_scale, growth_factor, backoff_factor, growth_interval)
        A.zero_async_begin(self.h, [g.data_ptr() for g in grads], sc, betas[0], betas[1],
                           self.stream.cuda_stream)

    def step_async(self, *, lr=1e-3, betas=(0.9, 0.999), eps=1e-8, weight_decay=0.0) -> None:
        hp = A.zero_hyper(lr, betas[0], betas[1], eps, weight_decay)
        A.zero_step_async(self.h, hp, self.stream.cuda_stream)

    def end_async(self) -> dict:
        st = A.zero_async_end(self.h, self.stream.cuda_stream)
        return {"t": st.t, "skipped": st.skipped, "loss_scale": st.loss_scale,
                "good_steps": st.good_steps}

    def close(self) -> None:
        if self.h:
            A.zero_destroy(self.h)
            self.h = 0

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


class ZeroOffloadAdam:
    """The offloaded step (include/zero_offload.h): fp32 master, m, v in host
    memory and Adam on the host cores; the reduce and the fp16 write-back run
    on the GPU. PyTorch allocates the device workspace, the page-locked
    staging and the host state; libzero does the work."""

    def __init__(self, psi: int, nd: int, stage: int, master_init, param_bufs: Sequence[torch.Tensor], *,
                 rank_view: int = -1, tensors: Sequence[tuple[int, ...]] | None = None,
                 chunk_elems: int = 0, threads: int = 0, stream: torch.cuda.Stream | None = None):
        import os

        import numpy as np

        self.cfg = A.Config(psi, nd, stage, rank_view=rank_view, tensors=tensors)
        self.ledger = A.zero_offload_bytes(self.cfg, chunk_elems)
        self.nd = nd
        m0 = np.ascontiguousarray(master_init.cpu().numpy() if isinstance(master_init, torch.Tensor)
                                  else master_init, dtype=np.float32)
        self.stream = stream or torch.cuda.current_stream()
        E = self.ledger.state_elems
        self.device_ws = torch.empty(self.ledger.device_bytes, dtype=torch.uint8, device=self.stream.device)
        self.staging = torch.empty(self.ledger.host_staging_bytes, dtype=torch.uint8, pin_memory=True)
        self.host_state = torch.empty(3 * max(E, 1), dtype=torch.float32)
        self.param_bufs = list(param_bufs)
        threads = threads or len(os.sched_getaffinity(0))
        self.h = A.zero_offload_init(self.cfg, chunk_elems, self.device_ws.data_ptr(), self.ledger.device_bytes,
                                     self.staging.data_ptr(), self.ledger.host_staging_bytes,
                                     self.host_state.data_ptr(), m0.ctypes.data,
                                     [p.data_ptr() for p in self.param_bufs], min(threads, 256),
                                     self.stream.cuda_stream)

    def step(self, grads: Sequence[torch.Tensor] | Sequence[int], loss_scale: float, *, lr=1e-3,
             betas=(0.9, 0.999), eps=1e-8, weight_decay=0.0) -> bool:
        ptrs = [g if isinstance(g, int) else g.data_ptr() for g in grads]
        if len(ptrs) != self.nd:
            raise ValueError(f"expected {self.nd} gradient buffers, got {len(ptrs)}")
        hp = A.zero_hyper(lr, betas[0], betas[1], eps, weight_decay)
        return A.zero_offload_step(self.h, ptrs, loss_scale, hp, self.stream.cuda_stream) == A.ZERO_SKIPPED

    def gather_layer(self, unit: int, out: torch.Tensor) -> None:
        """Stage 3: the unit's full fp16 weights into `out` (on this object's stream)."""
        A.zero_offload_gather_layer(self.h, unit, out.data_ptr(), self.stream.cuda_stream)

    @property
    def t(self) -> int:
        return A.zero_offload_state(self.h)[3]

    def state(self) -> tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
        """Live host master, m, v (state order; views of the host state)."""
        E = self.ledger.state_elems
        return self.host_state[:E], self.host_state[E:2 * E], self.host_state[2 * E:3 * E]

    def state_dict(self) -> dict:
        w, m, v = self.state()
        return {"master": w.clone(), "m": m.clone(), "v": v.clone(), "t": self.t}

    def load_state_dict(self, sd: dict) -> None:
        E = self.ledger.state_elems
        xs = [sd["master"].contiguous(), sd["m"].contiguous(), sd["v"].contiguous()]
        for x in xs:
            if x.dtype != torch.float32 or x.is_cuda or x.numel() != E:
                raise ValueError("state tensors must be host float32 of ledger.state_elems elements")
        A.zero_offload_set_state(self.h, xs[0].data_ptr(), xs[1].data_ptr(), xs[2].data_ptr(), int(sd["t"]),
                                 self.stream.cuda_stream)

    def close(self) -> None:
        if self.h:
            A.zero_offload_destroy(self.h)
            self.h = 0

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
