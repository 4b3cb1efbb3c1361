"""The C-ABI library builds for sm_100a, loads and exports every declared
symbol, and rejects bad arguments before touching CUDA (CPU only)."""
import ctypes
import os
import re

import pytest
import torch

import expert_combine_b200 as eb

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe_boundary.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(\w+)\s*\(", text, flags=re.M)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for fn in ("moe_route", "norm_quant_nvfp4", "expert_combine", "residual_join",
               "expert_combine_join", "moe_dispatch", "moe_dispatch_workspace_size",
               "router_logits", "router_weight_prepare", "moe_route_norm_quant_kernels",
               "moe_boundary_supported", "mb_last_error", "mb_device_status"):
        assert fn in names


def test_library_exports_every_declared_symbol():
    lib = eb.load()
    for fn in declared_functions():
        assert hasattr(lib, fn), fn


def test_supported_predicate():
    assert eb.supported(eb.STAGE_ROUTE, 8, 0, 256, 8)
    assert eb.supported(eb.STAGE_ROUTE, 8, 0, 2560, 22)
    assert not eb.supported(eb.STAGE_ROUTE, 8, 0, 5000, 8)
    assert not eb.supported(eb.STAGE_ROUTE, 8, 0, 4, 8)
    assert not eb.supported(eb.STAGE_ROUTE, 8, 0, 256, 33)
    assert eb.supported(eb.STAGE_NORM_QUANT, 8, 4096, 0, 0, 4)
    assert not eb.supported(eb.STAGE_NORM_QUANT, 8, 4096, 0, 0, 3)
    assert not eb.supported(eb.STAGE_NORM_QUANT, 8, 32768, 0, 0, 1)
    assert eb.supported(eb.STAGE_COMBINE, 8, 8192, 0, 8)
    assert not eb.supported(eb.STAGE_COMBINE, 8, 8200, 0, 8)
    assert eb.supported(eb.STAGE_JOIN, 8, 16384)
    assert eb.supported(eb.STAGE_DISPATCH, 8192, 0, 256, 8)
    assert eb.supported(eb.STAGE_DISPATCH, 65536, 0, 4096, 32)
    assert not eb.supported(eb.STAGE_DISPATCH, 8, 0, 0, 8)
    assert not eb.supported(eb.STAGE_DISPATCH, 8, 0, 4097, 8)
    assert not eb.supported(eb.STAGE_DISPATCH, 1 << 27, 0, 256, 32)
    assert eb.supported(eb.STAGE_ROUTER_LOGITS, 128, 8192, 256)
    assert eb.supported(eb.STAGE_ROUTER_LOGITS, 128, 4096, 2560)
    assert not eb.supported(eb.STAGE_ROUTER_LOGITS, 128, 8200, 256)
    assert not eb.supported(eb.STAGE_ROUTER_LOGITS, 128, 8192, 250)
    assert not eb.supported(99, 8, 16)


def test_route_norm_quant_kernels_query_without_device_work():
    assert eb.route_norm_quant_kernels(0, 8192, 256, 8) == 0
    assert eb.route_norm_quant_kernels(8192, 8192, 5000, 8) == -1     # E too large
    assert eb.route_norm_quant_kernels(8192, 8200, 256, 8) == -1      # H not a multiple of 16
    assert eb.route_norm_quant_kernels(8192, 4096, 256, 8, tp=3) == -1


def test_bad_arguments_are_rejected_before_any_launch():
    lib = eb.load()
    N = None
    assert lib.moe_route(N, N, N, -1, 256, 8, N, N, N) == 1
    assert lib.moe_route(N, N, N, 4, 256, 0, N, N, N) == 2
    assert lib.moe_route(N, N, N, 0, 256, 8, N, N, N) == 0          # empty: no launch
    assert lib.moe_route(N, N, N, 4, 256, 8, N, N, N) == 1
    assert "null" in eb.last_error()
    odd = ctypes.c_void_p(0x1004)
    assert lib.moe_route(odd, odd, odd, 4, 256, 8, odd, odd, N) == 1
    assert "aligned" in eb.last_error()
    assert lib.norm_quant_nvfp4(N, 4, 100, 1, N, 0.0, 1e-6, N, N, N, N) == 1
    assert lib.norm_quant_nvfp4(N, 4, 64, 3, N, 0.0, 1e-6, N, N, N, N) == 1
    assert lib.norm_quant_nvfp4(N, 0, 64, 1, N, 0.0, 1e-6, N, N, N, N) == 0
    assert lib.expert_combine(N, 10, 64, N, N, 4, 33, N, 0.0, 1e-6, N, N) == 2
    assert lib.expert_combine(N, -1, 64, N, N, 4, 8, N, 0.0, 1e-6, N, N) == 1
    assert lib.expert_combine(N, 10, 64, N, N, 0, 8, N, 0.0, 1e-6, N, N) == 0
    assert lib.residual_join(N, N, N, 1.0, 0.5, 1e-6, N, 1.0, 1e-6, N, 4, 64, N) == 1
    a = ctypes.c_void_p(0x1000)
    assert lib.residual_join(a, a, a, 1.0, 0.5, 1e-6, a, 1.0, 1e-6, N, 4, 64, N) == 1
    assert "both" in eb.last_error()
    # dispatch: sizes, pointers and the workspace are checked before any launch
    Z = ctypes.c_size_t(0)
    assert lib.moe_dispatch(N, 4, 8, 0, 0, N, N, N, N, Z, N) == 2
    assert lib.moe_dispatch(N, 4, 8, -1, 256, N, N, N, N, Z, N) == 1
    assert lib.moe_dispatch(N, 4, 8, 0, 256, N, N, N, N, Z, N) == 1
    assert "null" in eb.last_error()
    assert lib.moe_dispatch(a, 8192, 8, 0, 256, a, a, a, N, Z, N) == 1
    assert "workspace" in eb.last_error()
    need = eb.dispatch_workspace_size(8192, 8, 256)
    assert lib.moe_dispatch(a, 8192, 8, 0, 256, a, a, a, a, ctypes.c_size_t(need - 1), N) == 1
    assert lib.moe_dispatch(a, 8192, 8, 0, 256, a, a, a, odd, ctypes.c_size_t(need), N) == 1
    assert "aligned" in eb.last_error()
    # the no-allocation dispatch refuses bad arguments exactly as moe_dispatch
    # does, before its own size limit, and refuses too large inputs only then
    big = (65536, 32, 0, 4096)                  # needs more scratch than the fixed array holds
    assert lib.moe_dispatch_noalloc(N, *big, N, N, N, N) == 1
    assert "null" in eb.last_error() and "moe_dispatch_noalloc" in eb.last_error()
    assert lib.moe_dispatch_noalloc(a, 65536, 32, -1, 4096, a, a, a, N) == 1
    assert lib.moe_dispatch_noalloc(odd, *big, a, a, a, N) == 1
    assert "aligned" in eb.last_error()
    assert lib.moe_dispatch_noalloc(a, 4, 8, 0, 0, a, a, a, N) == 2
    assert lib.moe_dispatch_noalloc(a, *big, a, a, a, N) == 2
    assert "scratch" in eb.last_error()


def test_router_projection_arguments_checked_before_launch():
    lib = eb.load()
    N = None
    a = ctypes.c_void_p(0x1000)
    odd = ctypes.c_void_p(0x1004)
    assert lib.router_logits(N, 4, 8200, N, 256, 1.0, N, N) == 2
    assert lib.router_logits(N, -1, 8192, N, 256, 1.0, N, N) == 1
    assert lib.router_logits(N, 0, 8192, N, 256, 1.0, N, N) == 0          # empty: no launch
    assert lib.router_logits(N, 4, 8192, N, 256, 1.0, N, N) == 1
    assert lib.router_logits(a, 4, 8192, odd, 256, 1.0, a, N) == 1
    assert "aligned" in eb.last_error()
    assert lib.router_weight_prepare(N, 256, 8192, N, N) == 1
    assert lib.router_weight_prepare(a, 250, 8192, a, N) == 2


def test_dispatch_workspace_size():
    # one tile (<= 4096 entries) needs none; beyond, one count per tile and
    # expert plus the totals
    assert eb.dispatch_workspace_size(512, 8, 256) == 0
    assert eb.dispatch_workspace_size(0, 8, 256) == 0
    assert eb.dispatch_workspace_size(513, 8, 256) == (2 + 1) * 256 * 4
    assert eb.dispatch_workspace_size(8192, 8, 256) == (16 + 1) * 256 * 4
    assert eb.dispatch_workspace_size(65536, 22, 512) == (352 + 1) * 512 * 4


def test_binding_refuses_cpu_tensors():
    import torch
    x = torch.zeros(4, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        eb.norm_quant_nvfp4(x, 4, torch.zeros(64, dtype=torch.bfloat16), 0.0, 1e-6,
                            torch.ones(1))


def test_finalize_ar_sizes_without_device_work():
    assert eb.finalize_ar_workspace_size(4, 128, 8192) > 4 * 128 * 8192 * 2
    assert eb.finalize_ar_workspace_size(9, 128, 8192) == 0      # more ranks than the kernel takes
    assert eb.finalize_ar_workspace_size(4, 128, 8200) == 0      # H not a multiple of 16
    assert eb.finalize_ar_workspace_size(4, 0, 8192) == 0
    assert eb.supported(eb.STAGE_FINALIZE_AR, 128, 8192, 0, 8, 4)
    assert not eb.supported(eb.STAGE_FINALIZE_AR, 128, 8192, 0, 8, 9)
    assert not eb.supported(eb.STAGE_FINALIZE_AR, 128, 8192, 0, 33, 4)


def test_trace_context_nests_and_keeps_names():
    assert not eb.tracing()
    with eb.trace():
        assert eb.tracing()
        with eb.trace():
            assert eb.tracing()
        assert eb.tracing()
    assert not eb.tracing()
    assert eb.expert_combine.__name__ == "expert_combine" and eb.expert_combine.__doc__
    # inside a trace, a call that fails its argument checks still raises and closes its range
    with eb.trace():
        with pytest.raises((TypeError, ValueError)):
            eb.moe_route(torch.zeros(4, 8), torch.zeros(8), torch.zeros(4, dtype=torch.int32), 2)
