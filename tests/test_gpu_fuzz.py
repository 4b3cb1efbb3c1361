"""Seeded random shapes through the whole boundary on the GPU against the
oracle: hidden sizes from 16 to 16384 (multiples of 16, contiguous or
rank-block), expert counts from k to 4096, top-k from 1 to 32, both gain
centres, batches on both sides of the router arrangements' thresholds.  Each
case runs the router + norm-quant call, the combine with the join and next
prenorm, and the dispatch of the routing ids, and compares all outputs with
the oracle at the parity bar (ids, codes, scales, rows bit-exact; weights
1e-6 relative; BF16 outputs one step; residual 1e-5 relative)."""
import numpy as np
import pytest
import torch

import expert_combine_b200 as eb
import oracle
from expert_combine_b200 import synth

from parity import bf16_ulp_diff, check_join_outputs

pytestmark = pytest.mark.gpu


def _draw(rng):
    H = int(rng.choice([16, 48, 64, 272, 1024, 1040, 2048, 2688, 4096, 8192, 16384]))
    tps = [tp for tp in (1, 2, 3, 4, 8) if H % tp == 0 and (H // tp) % 16 == 0]
    tp = int(rng.choice(tps))
    E = int(rng.choice([8, 33, 64, 100, 256, 512, 2560, 4096]))
    k = int(rng.integers(1, min(32, E) + 1))
    # element budget keeps the oracle and the expert rows small
    t_max = max(1, min(3000, (1 << 23) // H, (1 << 25) // (H * k)))
    T = int(rng.choice([1, 2, 7, 64, 128, 889, 1500, 3000]))
    T = max(1, min(T, t_max))
    gc = float(rng.choice([0.0, 1.0]))
    return T, H, E, k, tp, gc


def _draw_fused(rng):
    """Shapes that take the router inside the norm-quant kernel (a batch above
    six tokens per SM, the wide row path, E <= 256)."""
    H = int(rng.choice([2048, 2688, 4096, 8192]))
    tps = [tp for tp in (1, 2, 4) if (H // tp) % 64 == 0]
    tp = int(rng.choice(tps))
    E = int(rng.choice([8, 33, 64, 100, 256]))
    k = int(rng.integers(1, max(1, min(32, E, (1 << 25) // (H * 889))) + 1))
    T = int(rng.integers(889, max(890, min(3000, (1 << 23) // H, (1 << 25) // (H * k))) + 1))
    gc = float(rng.choice([0.0, 1.0]))
    return T, H, E, k, tp, gc


CASES = [("any", s) for s in range(24)] + [("fused", s) for s in range(8)]


@pytest.mark.parametrize("kind,seed", CASES)
def test_random_shapes_match_the_oracle(cuda_dev, kind, seed):
    rng = np.random.default_rng(1000 + seed + (500 if kind == "fused" else 0))
    T, H, E, k, tp, gc = _draw(rng) if kind == "any" else _draw_fused(rng)
    case = synth.make_case("tiny", device=cuda_dev, seed=2000 + seed, T=T, H=H, E=E, k=k, tp=tp, gc=gc,
                           join=True)
    ids, w, packed, sf = eb.moe_route_norm_quant(case.logits, case.bias, case.mask, case.k, case.x,
                                                 case.norm_w, case.gc, case.eps, case.gs, tp=tp)
    r = case.residual.clone()
    out = torch.empty(T, H, dtype=torch.bfloat16, device=cuda_dev)
    _, p = eb.expert_combine_join(case.expert_out, case.R, case.row_idx, w, case.post_w, case.post_gc,
                                  case.eps, r, case.gain, case.alpha, case.beta, case.eps, case.next_w,
                                  case.next_gc, case.eps, out=out)
    offs, row_idx, row_token = eb.moe_dispatch(ids, E)
    torch.cuda.synchronize()
    shape = f"T={T} H={H} E={E} k={k} tp={tp} gc={gc}"

    ids_o, w_o = oracle.route(synth.host(case.logits), synth.host(case.bias), synth.host(case.mask), k)
    assert np.array_equal(synth.host(ids), ids_o), shape
    rel = np.abs(synth.host(w).astype(np.float64) - w_o) / np.maximum(np.abs(w_o), 1e-30)
    assert np.all(rel <= 1e-6), shape
    p_o, s_o = oracle.norm_quant(synth.host(case.x), T, H, tp, synth.host(case.norm_w), gc, case.eps,
                                 float(synth.host(case.gs)[0]))
    assert np.array_equal(synth.host(packed), p_o) and np.array_equal(synth.host(sf), s_o), shape

    G = case.guard
    branch_o = oracle.combine(synth.host(case.expert_buf)[G:], case.R, synth.host(case.row_idx), w_o,
                              synth.host(case.post_w), case.post_gc, case.eps)
    assert bf16_ulp_diff(synth.host(out), branch_o).max() <= 1, shape
    r_o, p_o2, n_o = oracle.join(synth.host(case.residual), branch_o, synth.host(case.gain), case.alpha, case.beta,
                                 case.eps, synth.host(case.next_w), case.next_gc, case.eps, return_normed=True)
    check_join_outputs(synth.host(r), synth.host(p), r_o, p_o2, n_o, case.beta)

    offs_o, row_idx_o, row_token_o = oracle.dispatch(synth.host(ids), 0, E)
    assert np.array_equal(synth.host(offs), offs_o), shape
    assert np.array_equal(synth.host(row_idx), row_idx_o), shape
    assert np.array_equal(synth.host(row_token), row_token_o), shape
    assert eb.device_status() == 0
