"""Every output of every full-size workload against the CPU oracle.

The four large workloads (decode 128 x 8192, prefill 8192 x 8192, large-E gate
32768 x 4096 with E = 2560 and the rank-block input, wide top-k 65536 x 1024
with E = 512, k = 22) run at their full sizes through the C ABI, in the call
sequence the benchmark times, and every token is compared with the oracle:

  - routing ids and order bit-exact, weights within 1e-6 relative (the count of
    weights that are not bit-identical is reported);
  - NVFP4 codes and scales bit-exact; the oracle's near-threshold cases (an FP32
    pre-quantisation value, or the scale's FP32 argument, within one ulp of a
    rounding threshold) are counted and reported in the test summary;
  - combine output and next prenorm within one BF16 step, the FP32 residual
    within 1e-5 relative or beta x one BF16 step of the normed term.

Wide top-k runs its stages end to end: the router's ids feed the dispatch, the
dispatch's rows feed the combine, the router's weights weight it (TensorRT-LLM
PR 21842, FC1 workload; lmdeploy PR 4835 "MoE gate v2", dispatch scan).
"""
import numpy as np
import pytest
import torch

import expert_combine_b200 as eb
import oracle
from expert_combine_b200 import synth

from parity import bf16_ulp_diff, check_join_outputs

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


def _route_all(case):
    ids_o, w_o = oracle.route(synth.host(case.logits), synth.host(case.bias), synth.host(case.mask), case.k)
    return ids_o, w_o


def _check_route(ids, w, ids_o, w_o, what):
    ids_g, w_g = synth.host(ids), synth.host(w)
    bad = np.argwhere(ids_g != ids_o)
    assert bad.size == 0, f"{what}: ids differ at {bad[:5]}"
    rel = np.abs(w_g.astype(np.float64) - w_o) / np.maximum(np.abs(w_o), 1e-30)
    assert np.all(rel <= 1e-6), f"{what}: weights rel err {rel.max()}"
    return int((w_g.view(np.uint32) != w_o.view(np.uint32)).sum())


def _check_nq(packed, sf, case, report_near, what):
    p_o, s_o, near = oracle.norm_quant(synth.host(case.x), case.T, case.H, case.tp, synth.host(case.norm_w),
                                       case.gc, case.eps, float(synth.host(case.gs)[0]), return_near=True)
    p_g, s_g = synth.host(packed), synth.host(sf)
    bad_p, bad_s = int((p_g != p_o).sum()), int((s_g != s_o).sum())
    report_near(what, near, case.T * case.H, case.T * case.H // 16, bad_p, bad_s)
    assert bad_p == 0 and bad_s == 0, (
        f"{what}: {bad_p} packed bytes and {bad_s} scales differ (oracle near-threshold: codes {near[0]}, "
        f"scales {near[1]})")


def _check_combine(out, case, row_idx_host, w_o, what):
    G = case.guard
    want = oracle.combine(synth.host(case.expert_buf)[G:], case.R, row_idx_host, w_o, synth.host(case.post_w),
                          case.post_gc, case.eps)
    d = bf16_ulp_diff(synth.host(out), want)
    assert d.max() <= 1, f"{what}: combine differs by {d.max()} BF16 steps at {np.argwhere(d > 1)[:5]}"
    return want


@pytest.mark.parametrize("name", ["prefill", "large_e"])
def test_full_size_every_token(cuda_dev, name, report_near):
    """The benchmark's step at full size: moe_route_norm_quant then
    expert_combine with the router's weights; plus the standalone router and
    norm-quant calls on the same inputs."""
    case = synth.make_case(name, device=cuda_dev)
    ids_o, w_o = _route_all(case)
    ids, w, packed, sf = eb.moe_route_norm_quant(case.logits, case.bias, case.mask, case.k, case.x, case.norm_w,
                                                 case.gc, case.eps, case.gs, tp=case.tp)
    out = eb.expert_combine(case.expert_out, case.R, case.row_idx, w, case.post_w, case.post_gc, case.eps)
    torch.cuda.synchronize()
    assert eb.device_status() == 0
    nonexact = _check_route(ids, w, ids_o, w_o, f"{name} moe_route_norm_quant")
    assert nonexact == 0, f"{name}: {nonexact} weights not bit-identical"
    _check_nq(packed, sf, case, report_near, name)
    _check_combine(out, case, synth.host(case.row_idx), w_o, name)

    # the standalone calls of the same stages
    ids2, w2 = eb.moe_route(case.logits, case.bias, case.mask, case.k)
    packed2, sf2 = eb.norm_quant_nvfp4(case.x, case.T, case.norm_w, case.gc, case.eps, case.gs, tp=case.tp)
    torch.cuda.synchronize()
    assert torch.equal(ids2, ids) and torch.equal(w2, w)
    assert torch.equal(packed2, packed) and torch.equal(sf2, sf)
    assert eb.device_status() == 0


def test_full_size_decode_every_token(cuda_dev, report_near):
    """Decode (128 x 8192): the pre-expert call, then the combine fused with the
    gated residual join and the next prenorm, all tokens."""
    case = synth.make_case("decode", device=cuda_dev)
    ids_o, w_o = _route_all(case)
    ids, w, packed, sf = eb.moe_route_norm_quant(case.logits, case.bias, case.mask, case.k, case.x, case.norm_w,
                                                 case.gc, case.eps, case.gs, tp=case.tp)
    r = case.residual.clone()
    out = torch.empty(case.T, case.H, dtype=torch.bfloat16, device=cuda_dev)
    _, p = eb.expert_combine_join(case.expert_out, case.R, case.row_idx, w, case.post_w, case.post_gc, case.eps,
                                  r, case.gain, case.alpha, case.beta, case.eps, case.next_w, case.next_gc,
                                  case.eps, out=out)
    torch.cuda.synchronize()
    assert eb.device_status() == 0
    assert _check_route(ids, w, ids_o, w_o, "decode") == 0
    _check_nq(packed, sf, case, report_near, "decode")
    branch_o = _check_combine(out, case, synth.host(case.row_idx), w_o, "decode")
    r_o, p_o, n_o = oracle.join(synth.host(case.residual), branch_o, synth.host(case.gain), case.alpha, case.beta,
                                case.eps, synth.host(case.next_w), case.next_gc, case.eps, return_normed=True)
    check_join_outputs(synth.host(r), synth.host(p), r_o, p_o, n_o, case.beta)


def test_full_size_wide_topk_end_to_end(cuda_dev, report_near):
    """Wide top-k (65536 x 1024, E = 512, k = 22), every stage end to end on
    the GPU: router + norm-quant, the dispatch of the router's ids, the combine
    over the dispatched rows with the router's weights; each stage against the
    oracle fed with the oracle's own previous stage."""
    case = synth.make_case("wide_topk", device=cuda_dev)
    T, k, E = case.T, case.k, case.E
    ids_o, w_o = _route_all(case)
    ids, w, packed, sf = eb.moe_route_norm_quant(case.logits, case.bias, case.mask, k, case.x, case.norm_w,
                                                 case.gc, case.eps, case.gs, tp=case.tp)
    offs, row_idx, row_token = eb.moe_dispatch(ids, E)
    out = eb.expert_combine(case.expert_out, case.R, row_idx, w, case.post_w, case.post_gc, case.eps)
    torch.cuda.synchronize()
    assert eb.device_status() == 0
    assert _check_route(ids, w, ids_o, w_o, "wide_topk") == 0
    _check_nq(packed, sf, case, report_near, "wide_topk")
    offs_o, row_idx_o, row_token_o = oracle.dispatch(ids_o, 0, E)
    assert np.array_equal(synth.host(offs), offs_o)
    assert np.array_equal(synth.host(row_idx), row_idx_o)
    assert np.array_equal(synth.host(row_token), row_token_o)
    assert int(offs_o[-1]) == int((synth.host(case.mask) != 0).sum()) * k <= case.R
    _check_combine(out, case, row_idx_o, w_o, "wide_topk")
