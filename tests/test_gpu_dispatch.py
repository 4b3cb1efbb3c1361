"""Dispatch (expert-grouped rows of the routing entries) on the GPU, through the
C ABI, against the oracle's counting sort on the same seeded ids.

Integer work: every output is compared bit for bit, at every size.
"""
import numpy as np
import pytest
import torch

import expert_combine_b200 as eb
import oracle
from expert_combine_b200 import synth

from parity import check_combine_rows

pytestmark = pytest.mark.gpu


def _run(ids_h, E, expert_begin, dev, workspace=None):
    ids = torch.from_numpy(ids_h).to(dev)
    off, idx, tok = eb.moe_dispatch(ids, E, expert_begin, workspace=workspace)
    torch.cuda.synchronize()
    return synth.host(off), synth.host(idx), synth.host(tok)


def _check(ids_h, E, expert_begin, dev):
    off, idx, tok = _run(ids_h, E, expert_begin, dev)
    o_off, o_idx, o_tok = oracle.dispatch(ids_h, expert_begin, E)
    assert np.array_equal(off, o_off)
    assert np.array_equal(idx, o_idx)
    assert np.array_equal(tok, o_tok)
    return off, idx, tok


# one tile (single kernel), tile boundaries, several tiles with a ragged tail
@pytest.mark.parametrize("T,k,E", [(1, 1, 1), (16, 8, 256), (128, 8, 256), (512, 8, 256), (513, 8, 256),
                                   (1000, 8, 256), (4096, 1, 7), (4097, 1, 7), (3000, 32, 4096),
                                   (777, 22, 512), (2048, 8, 2560)])
def test_dispatch_shapes(cuda_dev, T, k, E):
    ids = synth.make_topk_ids(T, k, E, seed=T * 31 + k, invalid_frac=0.01).numpy()
    _check(ids, E, 0, cuda_dev)


@pytest.mark.parametrize("name,T,k,E", [("prefill", 8192, 8, 256), ("large_e", 32768, 8, 2560),
                                        ("wide_topk", 65536, 22, 512)])
def test_dispatch_full_size(cuda_dev, name, T, k, E):
    """The workloads' shapes in full (the whole layout is compared)."""
    ids = synth.make_topk_ids(T, k, E, seed=synth.SEEDS[name], invalid_frac=0.01).numpy()
    _check(ids, E, 0, cuda_dev)


def test_dispatch_expert_parallel_range_and_repeats(cuda_dev):
    """Ids outside [expert_begin, expert_begin + E) get no row; repeated
    experts inside a token keep the flattened order."""
    ids = synth.make_topk_ids(5000, 8, 64, seed=7, span=200, distinct=False).numpy()
    ids[3, :] = 100           # one token, the same expert eight times
    _check(ids, 64, 100, cuda_dev)
    _check(ids, 64, 0, cuda_dev)


def test_dispatch_degenerate(cuda_dev):
    # nothing valid
    ids = np.full((6000, 4), -1, np.int32)
    off, idx, tok = _check(ids, 16, 0, cuda_dev)
    assert off[-1] == 0 and np.all(tok == -1)
    # every entry on one expert
    ids = np.zeros((3000, 2), np.int32)
    _check(ids, 1, 0, cuda_dev)
    # garbage ids far outside the range, including INT32 extremes
    ids = np.array([[np.iinfo(np.int32).min, 5], [np.iinfo(np.int32).max, 2]], np.int32)
    _check(ids, 8, 0, cuda_dev)
    # zero tokens: offsets are still written (all zero)
    off = torch.full((9,), 7, dtype=torch.int32, device=cuda_dev)
    eb.moe_dispatch(torch.empty(0, 8, dtype=torch.int32, device=cuda_dev), 8, expert_offsets=off)
    torch.cuda.synchronize()
    assert synth.host(off).tolist() == [0] * 9


def test_dispatch_repeat_calls_share_a_workspace(cuda_dev):
    """The workspace carries nothing between calls: two calls on different
    ids with one workspace both match the oracle, in either order."""
    E = 512
    a = synth.make_topk_ids(9000, 8, E, seed=1).numpy()
    b = synth.make_topk_ids(9000, 8, E, seed=2, masked_frac=0.5).numpy()
    ws = torch.empty(eb.dispatch_workspace_size(9000, 8, E), dtype=torch.uint8, device=cuda_dev)
    for ids in (a, b, a):
        off, idx, tok = _run(ids, E, 0, cuda_dev, workspace=ws)
        o = oracle.dispatch(ids, 0, E)
        assert np.array_equal(off, o[0]) and np.array_equal(idx, o[1]) and np.array_equal(tok, o[2])


def test_dispatch_graph_replay(cuda_dev):
    """Captured once, replayed on new ids written into the same buffers."""
    T, k, E = 6000, 8, 256
    ids = torch.from_numpy(synth.make_topk_ids(T, k, E, seed=3).numpy()).to(cuda_dev)
    off = torch.empty(E + 1, dtype=torch.int32, device=cuda_dev)
    idx = torch.empty(T, k, dtype=torch.int32, device=cuda_dev)
    tok = torch.empty(T * k, dtype=torch.int32, device=cuda_dev)
    ws = torch.empty(eb.dispatch_workspace_size(T, k, E), dtype=torch.uint8, device=cuda_dev)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        eb.moe_dispatch(ids, E, 0, off, idx, tok, ws)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        eb.moe_dispatch(ids, E, 0, off, idx, tok, ws)
    for seed in (4, 5):
        new = synth.make_topk_ids(T, k, E, seed=seed, masked_frac=0.2).numpy()
        ids.copy_(torch.from_numpy(new))
        g.replay()
        torch.cuda.synchronize()
        o = oracle.dispatch(new, 0, E)
        assert np.array_equal(synth.host(off), o[0]) and np.array_equal(synth.host(idx), o[1])
        assert np.array_equal(synth.host(tok), o[2])


def test_route_dispatch_combine_chain(cuda_dev):
    """Router -> dispatch -> combine on the GPU, each step's input taken from
    the previous GPU step, against the same chain of oracle steps on the host
    (expert outputs laid out in the dispatched row order)."""
    case = synth.make_case("tiny", device=cuda_dev, T=300, H=1024, E=64, k=8)
    ids, w = eb.moe_route(case.logits, case.bias, case.mask, case.k)
    off, idx, tok = eb.moe_dispatch(ids, case.E)
    torch.cuda.synchronize()
    ids_o, w_o = oracle.route(synth.host(case.logits), synth.host(case.bias), synth.host(case.mask), case.k)
    off_o, idx_o, tok_o = oracle.dispatch(ids_o, 0, case.E)
    assert np.array_equal(synth.host(ids), ids_o)
    assert np.array_equal(synth.host(off), off_o)
    assert np.array_equal(synth.host(idx), idx_o)
    assert np.array_equal(synth.host(tok), tok_o)
    R = int(off_o[-1])
    # expert outputs for the R dispatched rows (seeded, BF16)
    gen = torch.Generator(device="cpu")
    gen.manual_seed(99)
    rows = torch.randn(R, case.H, generator=gen).to(torch.bfloat16).to(cuda_dev)
    out = eb.expert_combine(rows, R, idx, w, case.post_w, case.post_gc, case.eps)
    torch.cuda.synchronize()
    check_combine_rows(synth.host(out), synth.host(rows), R, idx_o, w_o, synth.host(case.post_w),
                       case.post_gc, case.eps)
