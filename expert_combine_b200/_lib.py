"""ctypes binding of libmoe_boundary.so (argument marshalling only)."""
from __future__ import annotations

import ctypes
import os
import threading
from typing import Optional

import torch

from . import build as _build

# ---------------------------------------------------------------------------- NVTX ranges
# Off by default (no cost beyond one flag test per call).  Inside `trace()`,
# every call of the binding is an NVTX range named after its C entry point,
# so a profiler's timeline (or `ncu --nvtx --nvtx-include`) can pick out the
# boundary's kernels by call.
_trace_depth = 0


class trace:
    """Context manager: NVTX ranges around every call of the library while active."""

    def __enter__(self):
        global _trace_depth
        _trace_depth += 1
        return self

    def __exit__(self, *exc):
        global _trace_depth
        _trace_depth -= 1
        return False


def tracing() -> bool:
    return _trace_depth > 0


def _traced(fn):
    name = fn.__name__

    def wrapper(*args, **kwargs):
        if _trace_depth <= 0:
            return fn(*args, **kwargs)
        torch.cuda.nvtx.range_push(name)
        try:
            return fn(*args, **kwargs)
        finally:
            torch.cuda.nvtx.range_pop()

    wrapper.__name__ = name
    wrapper.__qualname__ = fn.__qualname__
    wrapper.__doc__ = fn.__doc__
    wrapper.__wrapped__ = fn
    return wrapper

STAGE_ROUTE = 0
STAGE_NORM_QUANT = 1
STAGE_COMBINE = 2
STAGE_JOIN = 3
STAGE_COMBINE_JOIN = 4
STAGE_ROUTE_NORM_QUANT = 5
STAGE_DISPATCH = 6
STAGE_ROUTER_LOGITS = 7
STAGE_FINALIZE_AR = 8
FAR_MAX_WORLD = 8
IPC_HANDLE_BYTES = 64

_lock = threading.Lock()
_lib = None


class MoEBoundaryError(RuntimeError):
    """A library call returned an error status."""

    def __init__(self, fn: str, status: int, message: str):
        super().__init__(f"{fn} failed with status {status}: {message}")
        self.status = status


def lib_path() -> str:
    return _build.LIB


def load() -> ctypes.CDLL:
    """Load the library, building it first when it is missing or stale.

    Raises when it can be neither found nor built: there is no fallback path.
    """
    global _lib
    with _lock:
        if _lib is None:
            path = _build.LIB
            if _build.is_stale():
                try:
                    _build.build()
                except Exception as exc:   # no nvcc, compile error, ...
                    if not os.path.exists(path):
                        raise RuntimeError(
                            f"libmoe_boundary.so is missing and could not be built: {exc}") from exc
            lib = ctypes.CDLL(path)
            P, i32, i64, f32 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float
            sigs = {
                "moe_route": [P, P, P, i32, i32, i32, P, P, P],
                "moe_route_check_fast_sigmoid": [P, P],
                "norm_quant_nvfp4": [P, i32, i32, i32, P, f32, f32, P, P, P, P],
                "expert_combine": [P, i64, i32, P, P, i32, i32, P, f32, f32, P, P],
                "residual_join": [P, P, P, f32, f32, f32, P, f32, f32, P, i32, i32, P],
                "expert_combine_join": [P, i64, i32, P, P, i32, i32, P, f32, f32, P, P, P, f32, f32,
                                        f32, P, f32, f32, P, P],
                "moe_route_norm_quant": [P, P, P, i32, i32, P, P, P, i32, i32, i32, P, f32, f32, P, P,
                                         P, P],
                "moe_dispatch": [P, i32, i32, i32, i32, P, P, P, P, ctypes.c_size_t, P],
                "moe_dispatch_noalloc": [P, i32, i32, i32, i32, P, P, P, P],
                "router_logits": [P, i32, i32, P, i32, f32, P, P],
                "router_weight_prepare": [P, i32, i32, P, P],
                "moe_boundary_supported": [i32, i32, i32, i32, i32, i32],
                "moe_route_norm_quant_kernels": [i32, i32, i32, i32, i32],
                "finalize_ar_workspace_init": [P, i32, i32, i32, P],
                "expert_finalize_allreduce": [P, i64, i32, P, P, i32, i32, P, f32, f32, P, i32, i32, i32, P, P],
                "expert_finalize_allreduce_local": [P, P, i32, P, P, i32, i32, P, f32, f32, P, i32, i32, P, P],
                "mb_ipc_alloc": [ctypes.c_size_t, P],
                "mb_ipc_free": [P],
                "mb_ipc_get_handle": [P, P],
                "mb_ipc_open": [P, P],
                "mb_ipc_close": [P],
                "mb_last_error": [],
                "mb_device_status": [],
            }
            for name, args in sigs.items():
                fn = getattr(lib, name)
                fn.argtypes = args
                fn.restype = ctypes.c_char_p if name == "mb_last_error" else ctypes.c_int
            lib.moe_dispatch_workspace_size.argtypes = [i32, i32, i32]
            lib.moe_dispatch_workspace_size.restype = ctypes.c_size_t
            lib.finalize_ar_workspace_size.argtypes = [i32, i32, i32]
            lib.finalize_ar_workspace_size.restype = ctypes.c_size_t
            _lib = lib
    return _lib


def last_error() -> str:
    return load().mb_last_error().decode()


def _check(fn: str, status: int) -> None:
    if status != 0:
        raise MoEBoundaryError(fn, status, last_error())


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _want(t: torch.Tensor, dtype: torch.dtype, name: str) -> None:
    if t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name}: expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name}: expected a contiguous tensor")


def supported(stage: int, T: int = 1, H: int = 16, E: int = 1, k: int = 1, tp: int = 1) -> bool:
    return bool(load().moe_boundary_supported(stage, T, H, E, k, tp))


def device_status() -> int:
    """Read and clear the library's device-side timeout flags (0 = none)."""
    v = load().mb_device_status()
    if v < 0:
        raise MoEBoundaryError("mb_device_status", v, last_error())
    return v


@_traced
def moe_route(logits: torch.Tensor, bias: torch.Tensor, token_mask: torch.Tensor, k: int,
              topk_ids: Optional[torch.Tensor] = None, topk_weights: Optional[torch.Tensor] = None,
              stream=None):
    """Sigmoid router gate -> (topk_ids int32 [T, k], topk_weights float32 [T, k])."""
    _want(logits, torch.float32, "logits")
    _want(bias, torch.float32, "bias")
    _want(token_mask, torch.uint8, "token_mask")
    T, E = logits.shape
    if topk_ids is None:
        topk_ids = torch.empty(T, k, dtype=torch.int32, device=logits.device)
    if topk_weights is None:
        topk_weights = torch.empty(T, k, dtype=torch.float32, device=logits.device)
    _want(topk_ids, torch.int32, "topk_ids")
    _want(topk_weights, torch.float32, "topk_weights")
    if bias.numel() != E or token_mask.numel() != T or topk_ids.shape != (T, k) \
            or topk_weights.shape != (T, k):
        raise ValueError("moe_route: shape mismatch")
    _check("moe_route", load().moe_route(_ptr(logits), _ptr(bias), _ptr(token_mask), T, E, k,
                                         _ptr(topk_ids), _ptr(topk_weights), _stream(stream)))
    return topk_ids, topk_weights


@_traced
def moe_route_check_fast_sigmoid(stream=None) -> float:
    """Largest |fast - exact| sigmoid over every binary32 input, measured on the
    device (the bound moe_route's shortlist relies on); synchronises."""
    dev = torch.device("cuda", torch.cuda.current_device())
    out = torch.empty(1, dtype=torch.float32, device=dev)
    _check("moe_route_check_fast_sigmoid", load().moe_route_check_fast_sigmoid(_ptr(out), _stream(stream)))
    torch.cuda.synchronize(dev)
    return float(out.item())


# The bound moe_route's shortlist assumes (MB_ROUTE_FAST_SIGMOID_BOUND).
ROUTE_FAST_SIGMOID_BOUND = 2.0 ** -21


@_traced
def norm_quant_nvfp4(x: torch.Tensor, num_tokens: int, norm_w: torch.Tensor, gain_center: float,
                     eps: float, global_scale: torch.Tensor, tp: int = 1,
                     packed: Optional[torch.Tensor] = None, sf: Optional[torch.Tensor] = None,
                     stream=None):
    """RMSNorm + NVFP4 -> (packed uint8 [M, H/2], sf uint8 [M, H/16]).

    ``x`` is [M, H] (tp == 1) or the rank-block [tp, M, H/tp] (any shape with
    M * H elements in that order).
    """
    _want(x, torch.bfloat16, "x")
    _want(norm_w, torch.bfloat16, "norm_w")
    _want(global_scale, torch.float32, "global_scale")
    H = norm_w.numel()
    M = int(num_tokens)
    if x.numel() != M * H:
        raise ValueError("norm_quant_nvfp4: x must hold num_tokens * H elements")
    if packed is None:
        packed = torch.empty(M, H // 2, dtype=torch.uint8, device=x.device)
    if sf is None:
        sf = torch.empty(M, H // 16, dtype=torch.uint8, device=x.device)
    _want(packed, torch.uint8, "packed")
    _want(sf, torch.uint8, "sf")
    if packed.numel() != M * (H // 2) or sf.numel() != M * (H // 16):
        raise ValueError("norm_quant_nvfp4: output shape mismatch")
    _check("norm_quant_nvfp4",
           load().norm_quant_nvfp4(_ptr(x), M, H, tp, _ptr(norm_w), float(gain_center), float(eps),
                                   _ptr(global_scale), _ptr(packed), _ptr(sf), _stream(stream)))
    return packed, sf


@_traced
def moe_route_norm_quant(logits: torch.Tensor, bias: torch.Tensor, token_mask: torch.Tensor, k: int,
                         x: torch.Tensor, norm_w: torch.Tensor, gain_center: float, eps: float,
                         global_scale: torch.Tensor, tp: int = 1,
                         topk_ids: Optional[torch.Tensor] = None,
                         topk_weights: Optional[torch.Tensor] = None,
                         packed: Optional[torch.Tensor] = None, sf: Optional[torch.Tensor] = None,
                         stream=None):
    """Router gate and RMSNorm + NVFP4 of the same tokens in one launch.

    -> (topk_ids, topk_weights, packed, sf), equal to moe_route + norm_quant_nvfp4.
    """
    _want(logits, torch.float32, "logits")
    _want(bias, torch.float32, "bias")
    _want(token_mask, torch.uint8, "token_mask")
    _want(x, torch.bfloat16, "x")
    _want(norm_w, torch.bfloat16, "norm_w")
    _want(global_scale, torch.float32, "global_scale")
    T, E = logits.shape
    H = norm_w.numel()
    if x.numel() != T * H or bias.numel() != E or token_mask.numel() != T:
        raise ValueError("moe_route_norm_quant: shape mismatch")
    dev = logits.device
    if topk_ids is None:
        topk_ids = torch.empty(T, k, dtype=torch.int32, device=dev)
    if topk_weights is None:
        topk_weights = torch.empty(T, k, dtype=torch.float32, device=dev)
    if packed is None:
        packed = torch.empty(T, H // 2, dtype=torch.uint8, device=dev)
    if sf is None:
        sf = torch.empty(T, H // 16, dtype=torch.uint8, device=dev)
    for t, dt, name in ((topk_ids, torch.int32, "topk_ids"), (topk_weights, torch.float32, "topk_weights"),
                        (packed, torch.uint8, "packed"), (sf, torch.uint8, "sf")):
        _want(t, dt, name)
    _check("moe_route_norm_quant",
           load().moe_route_norm_quant(_ptr(logits), _ptr(bias), _ptr(token_mask), E, k,
                                       _ptr(topk_ids), _ptr(topk_weights), _ptr(x), T, H, tp,
                                       _ptr(norm_w), float(gain_center), float(eps),
                                       _ptr(global_scale), _ptr(packed), _ptr(sf), _stream(stream)))
    return topk_ids, topk_weights, packed, sf



def route_norm_quant_kernels(M: int, H: int, E: int, k: int, tp: int = 1) -> int:
    """Kernels ``moe_route_norm_quant`` enqueues for these sizes on the current
    device (for a 16-byte-aligned x); -1 when unsupported or without a device."""
    return int(load().moe_route_norm_quant_kernels(M, H, tp, E, k))

@_traced
def expert_combine(expert_out: torch.Tensor, num_rows: int, row_idx: torch.Tensor,
                   weights: torch.Tensor, norm_w: torch.Tensor, gain_center: float, eps: float,
                   out: Optional[torch.Tensor] = None, stream=None):
    """Post-expert RMSNorm + weighted top-k combine -> out bf16 [T, H]."""
    _want(expert_out, torch.bfloat16, "expert_out")
    _want(row_idx, torch.int32, "row_idx")
    _want(weights, torch.float32, "weights")
    _want(norm_w, torch.bfloat16, "norm_w")
    H = norm_w.numel()
    T, k = row_idx.shape
    if weights.shape != (T, k) or expert_out.shape[-1] != H:
        raise ValueError("expert_combine: shape mismatch")
    if out is None:
        out = torch.empty(T, H, dtype=torch.bfloat16, device=row_idx.device)
    _want(out, torch.bfloat16, "out")
    _check("expert_combine",
           load().expert_combine(_ptr(expert_out), int(num_rows), H, _ptr(row_idx), _ptr(weights),
                                 T, k, _ptr(norm_w), float(gain_center), float(eps), _ptr(out),
                                 _stream(stream)))
    return out


@_traced
def residual_join(residual: torch.Tensor, branch: torch.Tensor, gain: torch.Tensor, alpha: float,
                  beta: float, eps: float, next_w: Optional[torch.Tensor] = None,
                  next_gc: float = 1.0, next_eps: float = 1e-6,
                  next_prenorm: Optional[torch.Tensor] = None, stream=None):
    """Gated residual join (residual updated in place) -> next_prenorm or None."""
    _want(residual, torch.float32, "residual")
    _want(branch, torch.bfloat16, "branch")
    _want(gain, torch.bfloat16, "gain")
    T, H = residual.shape
    if branch.shape != (T, H) or gain.numel() != H:
        raise ValueError("residual_join: shape mismatch")
    if next_w is not None:
        _want(next_w, torch.bfloat16, "next_w")
        if next_prenorm is None:
            next_prenorm = torch.empty(T, H, dtype=torch.bfloat16, device=residual.device)
        _want(next_prenorm, torch.bfloat16, "next_prenorm")
    _check("residual_join",
           load().residual_join(_ptr(residual), _ptr(branch), _ptr(gain), float(alpha),
                                float(beta), float(eps), _ptr(next_w), float(next_gc),
                                float(next_eps), _ptr(next_prenorm), T, H, _stream(stream)))
    return next_prenorm


@_traced
def expert_combine_join(expert_out: torch.Tensor, num_rows: int, row_idx: torch.Tensor,
                        weights: torch.Tensor, norm_w: torch.Tensor, gain_center: float,
                        eps: float, residual: torch.Tensor, gain: torch.Tensor, alpha: float,
                        beta: float, join_eps: float, next_w: Optional[torch.Tensor] = None,
                        next_gc: float = 1.0, next_eps: float = 1e-6,
                        out: Optional[torch.Tensor] = None,
                        next_prenorm: Optional[torch.Tensor] = None, stream=None):
    """Combine fused with the residual join -> (out or None, next_prenorm or None)."""
    _want(expert_out, torch.bfloat16, "expert_out")
    _want(row_idx, torch.int32, "row_idx")
    _want(weights, torch.float32, "weights")
    _want(norm_w, torch.bfloat16, "norm_w")
    _want(residual, torch.float32, "residual")
    _want(gain, torch.bfloat16, "gain")
    H = norm_w.numel()
    T, k = row_idx.shape
    if weights.shape != (T, k) or residual.shape != (T, H) or gain.numel() != H:
        raise ValueError("expert_combine_join: shape mismatch")
    if out is not None:
        _want(out, torch.bfloat16, "out")
    if next_w is not None:
        _want(next_w, torch.bfloat16, "next_w")
        if next_prenorm is None:
            next_prenorm = torch.empty(T, H, dtype=torch.bfloat16, device=residual.device)
    _check("expert_combine_join",
           load().expert_combine_join(_ptr(expert_out), int(num_rows), H, _ptr(row_idx),
                                      _ptr(weights), T, k, _ptr(norm_w), float(gain_center),
                                      float(eps), _ptr(out), _ptr(residual), _ptr(gain),
                                      float(alpha), float(beta), float(join_eps), _ptr(next_w),
                                      float(next_gc), float(next_eps), _ptr(next_prenorm),
                                      _stream(stream)))
    return out, next_prenorm


def dispatch_workspace_size(T: int, k: int, E: int) -> int:
    """Bytes of device workspace moe_dispatch needs for T tokens x k picks over E experts."""
    return int(load().moe_dispatch_workspace_size(T, k, E))


@_traced
def moe_dispatch(topk_ids: torch.Tensor, num_experts: int, expert_begin: int = 0,
                 expert_offsets: Optional[torch.Tensor] = None, row_idx: Optional[torch.Tensor] = None,
                 row_token: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                 stream=None):
    """Expert-grouped rows of the routing entries ->
    (expert_offsets int32 [E + 1], row_idx int32 [T, k], row_token int32 [T * k]).

    ``workspace`` is a uint8 CUDA tensor of at least ``dispatch_workspace_size``
    bytes; when omitted, one is allocated here (the library itself never
    allocates)."""
    _want(topk_ids, torch.int32, "topk_ids")
    T, k = topk_ids.shape
    E = int(num_experts)
    dev = topk_ids.device
    if expert_offsets is None:
        expert_offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    if row_idx is None:
        row_idx = torch.empty(T, k, dtype=torch.int32, device=dev)
    if row_token is None:
        row_token = torch.empty(T * k, dtype=torch.int32, device=dev)
    _want(expert_offsets, torch.int32, "expert_offsets")
    _want(row_idx, torch.int32, "row_idx")
    _want(row_token, torch.int32, "row_token")
    if expert_offsets.numel() != E + 1 or row_idx.shape != (T, k) or row_token.numel() != T * k:
        raise ValueError("moe_dispatch: shape mismatch")
    need = dispatch_workspace_size(T, k, E)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    if workspace is not None:
        _want(workspace, torch.uint8, "workspace")
    ws_bytes = 0 if workspace is None else workspace.numel()
    _check("moe_dispatch", load().moe_dispatch(_ptr(topk_ids), T, k, int(expert_begin), E,
                                               _ptr(expert_offsets), _ptr(row_idx), _ptr(row_token),
                                               _ptr(workspace), ws_bytes, _stream(stream)))
    return expert_offsets, row_idx, row_token


@_traced
def moe_dispatch_noalloc(topk_ids: torch.Tensor, num_experts: int, expert_begin: int = 0,
                         expert_offsets: Optional[torch.Tensor] = None,
                         row_idx: Optional[torch.Tensor] = None,
                         row_token: Optional[torch.Tensor] = None, stream=None):
    """moe_dispatch with the library's fixed scratch array instead of a workspace,
    for callers that cannot allocate device memory on the calling path.

    Pass preallocated outputs to allocate nothing at all (outputs left as None
    are allocated here).  Calls that overlap on the GPU share the scratch and
    race; see the C header for the size limit."""
    _want(topk_ids, torch.int32, "topk_ids")
    T, k = topk_ids.shape
    E = int(num_experts)
    dev = topk_ids.device
    if expert_offsets is None:
        expert_offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    if row_idx is None:
        row_idx = torch.empty(T, k, dtype=torch.int32, device=dev)
    if row_token is None:
        row_token = torch.empty(T * k, dtype=torch.int32, device=dev)
    _want(expert_offsets, torch.int32, "expert_offsets")
    _want(row_idx, torch.int32, "row_idx")
    _want(row_token, torch.int32, "row_token")
    if expert_offsets.numel() != E + 1 or row_idx.shape != (T, k) or row_token.numel() != T * k:
        raise ValueError("moe_dispatch_noalloc: shape mismatch")
    _check("moe_dispatch_noalloc",
           load().moe_dispatch_noalloc(_ptr(topk_ids), T, k, int(expert_begin), E, _ptr(expert_offsets),
                                       _ptr(row_idx), _ptr(row_token), _stream(stream)))
    return expert_offsets, row_idx, row_token


@_traced
def router_weight_prepare(w: torch.Tensor, w3: Optional[torch.Tensor] = None, stream=None):
    """FP32 router weight [E, H] -> its three BF16 parts [3, E, H] (done once)."""
    _want(w, torch.float32, "w")
    E, H = w.shape
    if w3 is None:
        w3 = torch.empty(3, E, H, dtype=torch.bfloat16, device=w.device)
    _want(w3, torch.bfloat16, "w3")
    if w3.shape != (3, E, H):
        raise ValueError("router_weight_prepare: shape mismatch")
    _check("router_weight_prepare", load().router_weight_prepare(_ptr(w), E, H, _ptr(w3), _stream(stream)))
    return w3


@_traced
def router_logits(x: torch.Tensor, w3: torch.Tensor, scale: float = 1.0,
                  logits: Optional[torch.Tensor] = None, stream=None):
    """Router projection on the tensor cores: logits float32 [T, E] =
    scale * x [T, H] (BF16) @ w^T, w given as its prepared parts w3 [3, E, H]."""
    _want(x, torch.bfloat16, "x")
    _want(w3, torch.bfloat16, "w3")
    T, H = x.shape
    E = w3.shape[1]
    if w3.shape != (3, E, H):
        raise ValueError("router_logits: shape mismatch")
    if logits is None:
        logits = torch.empty(T, E, dtype=torch.float32, device=x.device)
    _want(logits, torch.float32, "logits")
    if logits.shape != (T, E):
        raise ValueError("router_logits: shape mismatch")
    _check("router_logits", load().router_logits(_ptr(x), T, H, _ptr(w3), E, float(scale), _ptr(logits),
                                                 _stream(stream)))
    return logits


# ---------------------------------------------------------------------------- finalize + all-reduce
def finalize_ar_workspace_size(world: int, T_max: int, H: int) -> int:
    """Bytes of one rank's finalize all-reduce workspace (0 when unsupported)."""
    return int(load().finalize_ar_workspace_size(world, T_max, H))


@_traced
def finalize_ar_workspace_init(workspace, world: int, T_max: int, H: int, stream=None) -> None:
    """Zero a workspace's call counter and flags (a tensor or a device address)."""
    ptr = _ptr(workspace) if isinstance(workspace, torch.Tensor) else ctypes.c_void_p(int(workspace))
    _check("finalize_ar_workspace_init",
           load().finalize_ar_workspace_init(ptr, world, T_max, H, _stream(stream)))


def _addr(x) -> int:
    return int(x.data_ptr()) if isinstance(x, torch.Tensor) else int(x)


def _far_rank_check(fn, expert_out, row_idx, weights, norm_w, out):
    _want(expert_out, torch.bfloat16, "expert_out")
    _want(row_idx, torch.int32, "row_idx")
    _want(weights, torch.float32, "weights")
    _want(out, torch.bfloat16, "out")
    H = norm_w.numel()
    T, k = row_idx.shape
    if expert_out.dim() != 2 or expert_out.shape[1] != H or weights.shape != (T, k) or out.shape != (T, H):
        raise ValueError(f"{fn}: shape mismatch")


@_traced
def expert_finalize_allreduce(expert_out: torch.Tensor, num_rows: int, row_idx: torch.Tensor,
                              weights: torch.Tensor, norm_w: torch.Tensor, gain_center: float, eps: float,
                              workspaces, rank: int, T_max: int, out: Optional[torch.Tensor] = None,
                              stream=None) -> torch.Tensor:
    """One rank's expert finalize + tensor-parallel all-reduce.

    ``workspaces``: every rank's workspace (tensors or device addresses as
    mapped in this process), in rank order.  Returns out bf16 [T, H], the same
    on every rank.
    """
    _want(norm_w, torch.bfloat16, "norm_w")
    T, k = row_idx.shape
    H = norm_w.numel()
    if out is None:
        out = torch.empty(T, H, dtype=torch.bfloat16, device=row_idx.device)
    _far_rank_check("expert_finalize_allreduce", expert_out, row_idx, weights, norm_w, out)
    world = len(workspaces)
    ws = (ctypes.c_void_p * world)(*[_addr(w) for w in workspaces])
    _check("expert_finalize_allreduce",
           load().expert_finalize_allreduce(_ptr(expert_out), int(num_rows), H, _ptr(row_idx), _ptr(weights), T, k,
                                            _ptr(norm_w), float(gain_center), float(eps),
                                            ctypes.cast(ws, ctypes.c_void_p), world, int(rank), int(T_max),
                                            _ptr(out), _stream(stream)))
    return out


@_traced
def expert_finalize_allreduce_local(expert_outs, num_rows, row_idx, weights, norm_w: torch.Tensor,
                                    gain_center: float, eps: float, workspaces, T_max: int, outs=None,
                                    stream=None):
    """All ranks of the exchange in one launch on this device (lists of one
    entry per rank).  Returns the ranks' outputs (equal to one another)."""
    _want(norm_w, torch.bfloat16, "norm_w")
    world = len(expert_outs)
    if not (len(num_rows) == len(row_idx) == len(weights) == len(workspaces) == world):
        raise ValueError("expert_finalize_allreduce_local: one entry per rank in every list")
    T, k = row_idx[0].shape
    H = norm_w.numel()
    if outs is None:
        outs = [torch.empty(T, H, dtype=torch.bfloat16, device=norm_w.device) for _ in range(world)]
    for r in range(world):
        if row_idx[r].shape != (T, k):
            raise ValueError("expert_finalize_allreduce_local: every rank's row_idx must be [T, k]")
        _far_rank_check("expert_finalize_allreduce_local", expert_outs[r], row_idx[r], weights[r], norm_w, outs[r])
    arr = lambda xs: (ctypes.c_void_p * world)(*[_addr(x) for x in xs])
    rows = (ctypes.c_int64 * world)(*[int(n) for n in num_rows])
    _check("expert_finalize_allreduce_local",
           load().expert_finalize_allreduce_local(
               ctypes.cast(arr(expert_outs), ctypes.c_void_p), ctypes.cast(rows, ctypes.c_void_p), H,
               ctypes.cast(arr(row_idx), ctypes.c_void_p), ctypes.cast(arr(weights), ctypes.c_void_p), T, k,
               _ptr(norm_w), float(gain_center), float(eps), ctypes.cast(arr(workspaces), ctypes.c_void_p), world,
               int(T_max), ctypes.cast(arr(outs), ctypes.c_void_p), _stream(stream)))
    return outs


# ---------------------------------------------------------------------------- peer memory (CUDA IPC)
def ipc_alloc(nbytes: int) -> int:
    p = ctypes.c_void_p()
    _check("mb_ipc_alloc", load().mb_ipc_alloc(int(nbytes), ctypes.byref(p)))
    return int(p.value)


def ipc_free(ptr: int) -> None:
    _check("mb_ipc_free", load().mb_ipc_free(ctypes.c_void_p(int(ptr))))


def ipc_get_handle(ptr: int) -> bytes:
    buf = ctypes.create_string_buffer(IPC_HANDLE_BYTES)
    _check("mb_ipc_get_handle", load().mb_ipc_get_handle(ctypes.c_void_p(int(ptr)), buf))
    return buf.raw


def ipc_open(handle: bytes) -> int:
    if len(handle) != IPC_HANDLE_BYTES:
        raise ValueError("ipc_open: a handle is 64 bytes")
    p = ctypes.c_void_p()
    _check("mb_ipc_open", load().mb_ipc_open(ctypes.create_string_buffer(handle, IPC_HANDLE_BYTES),
                                               ctypes.byref(p)))
    return int(p.value)


def ipc_close(ptr: int) -> None:
    _check("mb_ipc_close", load().mb_ipc_close(ctypes.c_void_p(int(ptr))))
