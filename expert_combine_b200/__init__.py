"""B200-native per-token MoE boundary: router gate, RMSNorm + NVFP4, dispatch, expert combine,
residual join.

Thin Python binding over the C ABI of ``libmoe_boundary.so`` (declared in
``include/moe_boundary.h``).  This package only marshals arguments: it checks
dtypes/devices, allocates outputs with torch when the caller passes none, and
enqueues the library call on torch's current CUDA stream.  Every step of the
boundary runs in the library's CUDA kernels; there is no host fallback.  If the
library cannot be loaded the calls raise.
"""
from __future__ import annotations

from ._lib import (  # noqa: F401
    FAR_MAX_WORLD,
    IPC_HANDLE_BYTES,
    MoEBoundaryError,
    ROUTE_FAST_SIGMOID_BOUND,
    STAGE_COMBINE,
    STAGE_COMBINE_JOIN,
    STAGE_DISPATCH,
    STAGE_FINALIZE_AR,
    STAGE_JOIN,
    STAGE_NORM_QUANT,
    STAGE_ROUTE,
    STAGE_ROUTE_NORM_QUANT,
    STAGE_ROUTER_LOGITS,
    device_status,
    dispatch_workspace_size,
    expert_combine,
    expert_combine_join,
    expert_finalize_allreduce,
    expert_finalize_allreduce_local,
    finalize_ar_workspace_init,
    finalize_ar_workspace_size,
    ipc_alloc,
    ipc_close,
    ipc_free,
    ipc_get_handle,
    ipc_open,
    last_error,
    lib_path,
    load,
    moe_dispatch,
    moe_dispatch_noalloc,
    moe_route,
    moe_route_check_fast_sigmoid,
    moe_route_norm_quant,
    norm_quant_nvfp4,
    residual_join,
    route_norm_quant_kernels,
    router_logits,
    router_weight_prepare,
    supported,
    trace,
    tracing,
)
