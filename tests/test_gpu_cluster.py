"""Few-token (decode) combine / join path -- one token per thread-block cluster,
the hidden dimension split across the cluster's CTAs -- against the oracle,
and against the row kernels that take more tokens.

Both paths follow the same canonical arithmetic, so the outputs are compared
bit for bit (the parity bar of one BF16 step / 1e-5 relative is not needed).
"""
import numpy as np
import pytest
import torch

import expert_combine_b200 as eb
import oracle
from expert_combine_b200 import synth

from parity import check_combine, check_join_outputs, oracle_combine

pytestmark = pytest.mark.gpu

SMS = 148   # B200


def cluster_max_tokens(H):
    """Largest T the cluster path takes at this H (one wave at 16 warps per SM)."""
    p2 = 1
    while p2 < H // 16:
        p2 <<= 1
    return (SMS * 512) // max(p2, 32)


@pytest.mark.parametrize("T", [1, 2, 7, 33, 64])
@pytest.mark.parametrize("H,k", [(16, 1), (48, 3), (512, 8), (1024, 22), (2688, 8), (8192, 8),
                                 (16384, 4), (4096, 32)])
def test_cluster_combine(cuda_dev, T, H, k):
    case = synth.make_case("tiny", device=cuda_dev, T=T, H=H, k=k, E=max(64, k), join=False)
    _, nonexact = check_combine(case)
    assert nonexact == 0


@pytest.mark.parametrize("T", [3, 64])
@pytest.mark.parametrize("H", [1024, 2688, 8192])
def test_cluster_combine_gain_centre_one(cuda_dev, T, H):
    case = synth.make_case("tiny", device=cuda_dev, T=T, H=H, join=False)
    g = torch.Generator(device="cpu")
    g.manual_seed(7)
    case.post_w.copy_((0.1 * torch.randn(H, generator=g)).to(torch.bfloat16))
    case.post_gc = 1.0
    _, nonexact = check_combine(case)
    assert nonexact == 0


def _join(case, branch, with_next):
    r = case.residual.clone()
    nw = case.next_w if with_next else None
    p = eb.residual_join(r, branch, case.gain, case.alpha, case.beta, case.eps, nw, case.next_gc, case.eps)
    torch.cuda.synchronize()
    return r, p


@pytest.mark.parametrize("T", [1, 5, 64])
@pytest.mark.parametrize("H", [64, 1024, 2688, 8192, 16384])
@pytest.mark.parametrize("with_next", [True, False])
def test_cluster_residual_join(cuda_dev, T, H, with_next):
    case = synth.make_case("tiny", device=cuda_dev, T=T, H=H, join=True)
    g = torch.Generator(device="cpu")
    g.manual_seed(3)
    branch = torch.randn(T, H, generator=g).to(torch.bfloat16).to(cuda_dev)
    r, p = _join(case, branch, with_next)
    r_o, p_o = oracle.join(synth.host(case.residual), synth.host(branch), synth.host(case.gain),
                           case.alpha, case.beta, case.eps, synth.host(case.next_w) if with_next else None,
                           case.next_gc, case.eps)
    assert np.array_equal(synth.host(r).view(np.uint32), r_o.view(np.uint32))
    if with_next:
        assert np.array_equal(synth.host(p), p_o)


@pytest.mark.parametrize("T,H,k", [(1, 8192, 8), (16, 8192, 8), (64, 8192, 8), (9, 2688, 22),
                                   (32, 16384, 32)])
def test_cluster_combine_join(cuda_dev, T, H, k):
    case = synth.make_case("decode", device=cuda_dev, T=T, H=H, k=k, E=max(64, k))
    r = case.residual.clone()
    out, p = eb.expert_combine_join(case.expert_out, case.R, case.row_idx, case.comb_wt, case.post_w,
                                    case.post_gc, case.eps, r, case.gain, case.alpha, case.beta, case.eps,
                                    case.next_w, case.next_gc, case.eps,
                                    out=torch.empty(T, H, dtype=torch.bfloat16, device=cuda_dev))
    torch.cuda.synchronize()
    branch_o = oracle_combine(case, synth.host(case.comb_wt))
    assert np.array_equal(synth.host(out), branch_o)
    r_o, p_o, n_o = oracle.join(synth.host(case.residual), branch_o, synth.host(case.gain), case.alpha,
                                case.beta, case.eps, synth.host(case.next_w), case.next_gc, case.eps,
                                return_normed=True)
    assert np.array_equal(synth.host(r).view(np.uint32), r_o.view(np.uint32))
    assert np.array_equal(synth.host(p), p_o)
    check_join_outputs(synth.host(r), synth.host(p), r_o, p_o, n_o, case.beta)


@pytest.mark.parametrize("H", [1024, 2688, 8192])
def test_cluster_and_row_paths_agree(cuda_dev, H):
    """The first 16 tokens of a batch large enough for the row kernels equal a
    16-token call on the same inputs (cluster path), for the fused combine +
    join."""
    T = 2400
    assert cluster_max_tokens(H) < T
    case = synth.make_case("decode", device=cuda_dev, T=T, H=H)
    outs = []
    for n in (T, 16):
        r = case.residual[:n].clone()
        out, p = eb.expert_combine_join(case.expert_out, case.R, case.row_idx[:n].contiguous(),
                                        case.comb_wt[:n].contiguous(), case.post_w, case.post_gc, case.eps,
                                        r, case.gain, case.alpha, case.beta, case.eps, case.next_w,
                                        case.next_gc, case.eps,
                                        out=torch.empty(n, H, dtype=torch.bfloat16, device=cuda_dev))
        torch.cuda.synchronize()
        outs.append((synth.host(out)[:16], synth.host(r)[:16], synth.host(p)[:16]))
    for a, b in zip(*outs):
        assert np.array_equal(a, b)


@pytest.mark.parametrize("H,k", [(16, 1), (48, 3), (1024, 22), (2688, 8), (8192, 8), (16384, 4)])
def test_row_path_small_batches(cuda_dev, H, k):
    """Just above the cluster path's largest batch: the row kernels."""
    T = cluster_max_tokens(H) + 1 + k
    case = synth.make_case("tiny", device=cuda_dev, T=T, H=H, k=k, E=max(64, k), join=False)
    tokens = np.unique(np.concatenate([np.arange(8), np.arange(T - 8, T), np.arange(0, T, 97)]))
    _, nonexact = check_combine(case, tokens=tokens)
    assert nonexact == 0


@pytest.mark.parametrize("H", [1024, 8192])
def test_cluster_largest_batch(cuda_dev, H):
    """The largest batch the cluster path takes, and one token more."""
    for T in (cluster_max_tokens(H), cluster_max_tokens(H) + 1):
        case = synth.make_case("tiny", device=cuda_dev, T=T, H=H, join=False)
        tokens = np.unique(np.concatenate([np.arange(4), np.arange(T - 4, T)]))
        _, nonexact = check_combine(case, tokens=tokens)
        assert nonexact == 0
