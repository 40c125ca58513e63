"""ZeRO stage 1/2/3 partitioned mixed-precision Adam step for B200 (sm_100a).

Nd data-parallel ranks are emulated as virtual ranks on one GPU. The work runs
in libzero.so (hand-written CUDA behind the C ABI in include/zero.h,
include/zero_offload.h and include/zero_peer.h); this package is the thin
Python binding (``_abi``), PyTorch-facing objects (``ZeroAdam``,
``ZeroOffloadAdam``; ``PeerRank``, rank r of a real job with one process per
GPU), the layer-gather prefetcher (``prefetch.LayerPrefetcher``) and the build
script. There is no CPU or eager fallback for the device step: if libzero.so
is missing, loading fails with an error.
"""
from . import _abi
from ._abi import (ZERO_ERR_ALIGN, ZERO_ERR_ARG, ZERO_ERR_CUDA, ZERO_ERR_INTERNAL,
                   ZERO_ERR_STAGE, ZERO_ERR_WORKSPACE, ZERO_OK, ZERO_PRECISION_BF16, ZERO_PRECISION_FP16,
                   ZERO_SKIPPED, ZERO_TENSOR_NO_DECAY, ZERO_VARIANT_FUSED, ZERO_VARIANT_FUSED_TMA,
                   ZERO_VARIANT_TWO_PASS, ZERO_VARIANT_TWO_PASS_TMA, Config, ZeroError, zero_current_state,
                   zero_destroy, zero_gather_layer, zero_init, zero_offload_bytes, zero_offload_destroy,
                   zero_offload_init, zero_offload_set_state, zero_offload_state, zero_offload_step,
                   zero_rank_shard, zero_state_bytes, zero_step, zero_step_commit, zero_step_launch,
                   zero_peer_close, zero_peer_export, zero_peer_open, zero_stream_copy, zero_unit_range)

__all__ = [
    "Config", "ZeroError", "ZeroAdam", "ZeroOffloadAdam", "zero_state_bytes", "zero_rank_shard",
    "zero_unit_range", "zero_init", "zero_step", "zero_step_launch", "zero_step_commit",
    "zero_gather_layer", "zero_current_state", "zero_stream_copy", "zero_destroy",
    "zero_offload_bytes", "zero_offload_init", "zero_offload_step", "zero_offload_state",
    "zero_offload_set_state", "zero_offload_destroy", "zero_peer_export", "zero_peer_open",
    "zero_peer_close", "PeerRank",
    "ZERO_OK", "ZERO_SKIPPED", "ZERO_ERR_ARG", "ZERO_ERR_ALIGN", "ZERO_ERR_STAGE",
    "ZERO_ERR_WORKSPACE", "ZERO_ERR_CUDA", "ZERO_ERR_INTERNAL", "ZERO_VARIANT_FUSED",
    "ZERO_VARIANT_TWO_PASS", "ZERO_VARIANT_FUSED_TMA", "ZERO_VARIANT_TWO_PASS_TMA",
    "ZERO_PRECISION_FP16", "ZERO_PRECISION_BF16", "ZERO_TENSOR_NO_DECAY",
]


def __getattr__(name):
    if name in ("ZeroAdam", "ZeroOffloadAdam"):
        from . import optimizer
        return getattr(optimizer, name)
    if name == "PeerRank":
        from . import distributed
        return distributed.PeerRank
    raise AttributeError(name)
