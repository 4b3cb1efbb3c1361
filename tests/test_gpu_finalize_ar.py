"""Expert finalize + tensor-parallel all-reduce on the GPU (all ranks of the
exchange in one launch on one device, through the C ABI) against the oracle:
every rank's output equal to the oracle's bit for bit, over world sizes,
widths, gain centres, repeated calls (the double-buffered exchange), CUDA
graph replay with changed inputs, and a wait that runs out when a rank never
arrives (the error is reported through mb_device_status, nothing hangs)."""
import numpy as np
import pytest
import torch

import expert_combine_b200 as eb
import oracle
from expert_combine_b200 import synth

pytestmark = pytest.mark.gpu


def _workspaces(world, T_max, H, dev):
    n = eb.finalize_ar_workspace_size(world, T_max, H)
    ws = [torch.empty(n, dtype=torch.uint8, device=dev) for _ in range(world)]
    for w in ws:
        eb.finalize_ar_workspace_init(w, world, T_max, H)
    return ws


def _oracle(c, weights=None):
    wt = synth.host(c.weights if weights is None else weights)
    out, _ = oracle.finalize_allreduce([synth.host(e) for e in c.expert_out], c.R,
                                       np.stack([synth.host(i) for i in c.row_idx]), wt, synth.host(c.norm_w),
                                       c.gc, c.eps)
    return out


def _local(c, ws, T_max, weights=None, outs=None):
    w = c.weights if weights is None else weights
    return eb.expert_finalize_allreduce_local(c.expert_out, c.R, c.row_idx, [w] * c.world, c.norm_w, c.gc, c.eps,
                                              ws, T_max, outs=outs)


@pytest.mark.parametrize("world,T,H,gc", [(1, 5, 64, 0.0), (2, 37, 1040, 1.0), (3, 16, 4096, 0.0),
                                          (4, 128, 8192, 1.0), (8, 33, 2048, 0.0), (4, 1, 8192, 0.0),
                                          (2, 130, 256, 1.0), (8, 64, 16384, 0.0), (4, 128, 8192, 0.0)])
def test_local_exchange_matches_oracle(cuda_dev, world, T, H, gc):
    c = synth.make_ep_case(T, H, 8, 256, world, seed=world * 100 + T, gc=gc, device=cuda_dev)
    ws = _workspaces(world, max(T, 8), H, cuda_dev)
    outs = _local(c, ws, max(T, 8))
    torch.cuda.synchronize()
    want = _oracle(c)
    for r in range(world):
        got = synth.host(outs[r])
        assert np.array_equal(got, want), f"rank {r}: {int((got != want).sum())} elements differ"
    assert eb.device_status() == 0


def test_repeated_calls_use_alternate_buffers(cuda_dev):
    """Six calls back to back, new weights each time, no synchronisation: each
    call's exchange uses its own epoch and buffer parity."""
    world, T, H = 4, 64, 1024
    c = synth.make_ep_case(T, H, 8, 64, world, seed=7, device=cuda_dev)
    ws = _workspaces(world, T, H, cuda_dev)
    g = torch.Generator(device="cpu")
    g.manual_seed(3)
    weights = [torch.rand(T, 8, generator=g).to(cuda_dev) for _ in range(6)]
    results = [_local(c, ws, T, weights=w) for w in weights]
    torch.cuda.synchronize()
    for w, outs in zip(weights, results):
        want = _oracle(c, w)
        for o in outs:
            assert np.array_equal(synth.host(o), want)
    assert eb.device_status() == 0


def test_graph_replay_with_changed_inputs(cuda_dev):
    """The call counter lives in the workspaces: a captured call replays
    correctly with its inputs changed in place, nothing set on the host."""
    world, T, H = 2, 32, 2048
    c = synth.make_ep_case(T, H, 8, 64, world, seed=9, device=cuda_dev)
    ws = _workspaces(world, T, H, cuda_dev)
    w = c.weights.clone()
    outs = [torch.empty(T, H, dtype=torch.bfloat16, device=cuda_dev) for _ in range(world)]
    _local(c, ws, T, weights=w, outs=outs)          # warm-up outside the capture
    torch.cuda.synchronize()
    s = torch.cuda.Stream(device=cuda_dev)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(graph, stream=s):
            _local(c, ws, T, weights=w, outs=outs)
    g = torch.Generator(device="cpu")
    g.manual_seed(5)
    for _ in range(3):
        w.copy_(torch.rand(T, 8, generator=g))
        graph.replay()
        torch.cuda.synchronize()
        want = _oracle(c, w)
        for o in outs:
            assert np.array_equal(synth.host(o), want)
    assert eb.device_status() == 0


def test_one_rank_entry_point(cuda_dev):
    """The per-process entry point with one rank equals the exchange."""
    T, H = 20, 4096
    c = synth.make_ep_case(T, H, 8, 64, 1, seed=11, device=cuda_dev)
    ws = _workspaces(1, T, H, cuda_dev)
    out = eb.expert_finalize_allreduce(c.expert_out[0], c.R[0], c.row_idx[0], c.weights, c.norm_w, c.gc, c.eps,
                                       ws, 0, T)
    torch.cuda.synchronize()
    assert np.array_equal(synth.host(out), _oracle(c))
    assert eb.device_status() == 0


def test_missing_rank_ends_in_a_reported_timeout(cuda_dev):
    """Rank 1 never calls: rank 0's wait for its partials runs out after the
    2 s limit, the kernel returns, bit 4 of the device status is set; after
    re-initialising the workspaces the exchange works again."""
    world, T, H = 2, 8, 1024
    c = synth.make_ep_case(T, H, 8, 64, world, seed=13, device=cuda_dev)
    ws = _workspaces(world, T, H, cuda_dev)
    eb.expert_finalize_allreduce(c.expert_out[0], c.R[0], c.row_idx[0], c.weights, c.norm_w, c.gc, c.eps, ws, 0, T)
    torch.cuda.synchronize()
    assert eb.device_status() & 16
    for w in ws:
        eb.finalize_ar_workspace_init(w, world, T, H)
    outs = _local(c, ws, T)
    torch.cuda.synchronize()
    for o in outs:
        assert np.array_equal(synth.host(o), _oracle(c))
    assert eb.device_status() == 0


def test_invalid_calls_raise(cuda_dev):
    world, T, H = 2, 8, 1024
    c = synth.make_ep_case(T, H, 8, 64, world, seed=17, device=cuda_dev)
    ws = _workspaces(world, 4, H, cuda_dev)
    with pytest.raises(eb.MoEBoundaryError):          # T above the workspaces' T_max
        _local(c, ws, 4)
    with pytest.raises(eb.MoEBoundaryError):          # rank outside the world
        eb.expert_finalize_allreduce(c.expert_out[0], c.R[0], c.row_idx[0], c.weights, c.norm_w, 0.0, 1e-6,
                                     ws, 2, 4)
    bad = [w[16:] for w in ws]                          # not 256-byte aligned
    with pytest.raises(eb.MoEBoundaryError):
        eb.expert_finalize_allreduce_local(c.expert_out, c.R, c.row_idx, [c.weights] * 2, c.norm_w, 0.0, 1e-6,
                                           bad, 16)
