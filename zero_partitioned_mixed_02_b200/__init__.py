"""ZeRO stage 1/2/3 partitioned mixed-precision Adam step for B200 (sm_100a).

Nd data-parallel ranks are emulated as virtual ranks on one GPU. The work runs
in libzero.so (hand-written CUDA behind the C ABI in include/zero.h); this
package is the thin Python binding (``_abi``), a PyTorch-facing object
(``ZeroAdam``) and the build script. There is no CPU or eager fallback: if
libzero.so is missing, loading fails with an error.
"""
from . import _abi
from ._abi import (ZERO_ERR_ALIGN, ZERO_ERR_ARG, ZERO_ERR_CUDA, ZERO_ERR_INTERNAL,
                   ZERO_ERR_STAGE, ZERO_ERR_WORKSPACE, ZERO_OK, ZERO_SKIPPED,
                   ZERO_VARIANT_FUSED, ZERO_VARIANT_FUSED_TMA, ZERO_VARIANT_TWO_PASS, Config, ZeroError, zero_current_state,
                   zero_destroy, zero_gather_layer, zero_init, zero_rank_shard, zero_state_bytes,
                   zero_step, zero_step_commit, zero_step_launch, zero_stream_copy,
                   zero_unit_range)

__all__ = [
    "Config", "ZeroError", "ZeroAdam", "zero_state_bytes", "zero_rank_shard", "zero_unit_range",
    "zero_init", "zero_step", "zero_step_launch", "zero_step_commit", "zero_gather_layer", "zero_current_state", "zero_stream_copy",
    "zero_destroy", "ZERO_OK", "ZERO_SKIPPED", "ZERO_ERR_ARG", "ZERO_ERR_ALIGN", "ZERO_ERR_STAGE",
    "ZERO_ERR_WORKSPACE", "ZERO_ERR_CUDA", "ZERO_ERR_INTERNAL", "ZERO_VARIANT_FUSED",
    "ZERO_VARIANT_TWO_PASS", "ZERO_VARIANT_FUSED_TMA",
]


def __getattr__(name):
    if name == "ZeroAdam":
        from .optimizer import ZeroAdam
        return ZeroAdam
    raise AttributeError(name)
