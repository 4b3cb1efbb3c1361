"""moe_dispatch_noalloc: the dispatch for callers that cannot allocate device
memory (their memory belongs to an allocator they cannot reach from the call
site, or cudaMalloc's possible device-wide synchronisation is not acceptable on
their hot path).  It takes its scratch from a fixed array inside the library
instead of a caller workspace.

Called through the C ABI (ctypes on the loaded library) with preallocated
outputs, two calls in a row on different inputs, each compared with the
workspace entry point moe_dispatch on the same ids and with the CPU oracle's
counting sort.  The dispatch is integer work, so the comparison is exact.
This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

import expert_combine_b200 as eb
import oracle
from expert_combine_b200 import synth

pytestmark = pytest.mark.gpu


def _outputs(T, k, E, dev):
    return (torch.full((E + 1,), -7, dtype=torch.int32, device=dev),
            torch.full((T, k), -7, dtype=torch.int32, device=dev),
            torch.full((T * k,), -7, dtype=torch.int32, device=dev))


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


@pytest.mark.parametrize("T,k,E", [(8192, 8, 256), (32768, 8, 2560), (300, 8, 256)])
def test_noalloc_dispatch_equals_workspace_dispatch(cuda_dev, T, k, E):
    lib = eb.load()
    need = eb.dispatch_workspace_size(T, k, E)
    ws = torch.empty(max(need, 16), dtype=torch.uint8, device=cuda_dev)
    for seed in (21, 22):   # two calls in a row, different ids
        ids = synth.make_topk_ids(T, k, E, seed=seed * 1000 + T, invalid_frac=0.01).to(cuda_dev)
        want = _outputs(T, k, E, cuda_dev)
        got = _outputs(T, k, E, cuda_dev)
        st = lib.moe_dispatch(_p(ids), T, k, 0, E, *[_p(t) for t in want], _p(ws), ctypes.c_size_t(ws.numel()),
                              _stream())
        assert st == 0, eb.last_error()
        st = lib.moe_dispatch_noalloc(_p(ids), T, k, 0, E, *[_p(t) for t in got], _stream())
        assert st == 0, eb.last_error()
        torch.cuda.synchronize()
        for g, w in zip(got, want):
            assert np.array_equal(synth.host(g), synth.host(w))
        for g, o in zip(got, oracle.dispatch(synth.host(ids), 0, E)):
            assert np.array_equal(synth.host(g).reshape(o.shape), o)
    assert eb.device_status() == 0


def test_noalloc_dispatch_rejects_inputs_beyond_its_array(cuda_dev):
    lib = eb.load()
    T, k, E = 65536, 32, 4096           # needs 513 * 4096 * 4 bytes of scratch, above 1 MiB
    assert eb.dispatch_workspace_size(T, k, E) > (1 << 20)
    a = ctypes.c_void_p(0x1000)
    st = lib.moe_dispatch_noalloc(a, T, k, 0, E, a, a, a, _stream())
    assert st == 2
    assert "scratch" in eb.last_error()
