"""CUDA path (through the C ABI) against the CPU oracle on the same seeded inputs.

Every case here is compared in full (the full-size workloads are in
test_gpu_full_size.py).  The bar: routing ids and NVFP4 codes/scales
bit-exact, routing weights within 1e-6 relative, combine and prenorm within one
BF16 step, the FP32 residual within 1e-5 relative or beta x one BF16 step of
the normed term.
"""
import numpy as np
import pytest
import torch

import expert_combine_b200 as eb
import oracle
from expert_combine_b200 import synth

from parity import (bf16_ulp_diff, check_combine, check_join_outputs, check_norm_quant,
                    check_route, oracle_combine)

pytestmark = pytest.mark.gpu


# ------------------------------------------------------------------ small, in full
def test_tiny_all_stages(cuda_dev, report_near):
    case = synth.make_case("tiny", device=cuda_dev)
    ids, w, nonexact_w = check_route(case)
    assert nonexact_w == 0
    _, _, near = check_norm_quant(case)
    report_near("tiny", near, case.T * case.H, case.T * case.H // 16)
    _, nonexact = check_combine(case)
    assert nonexact == 0


@pytest.mark.parametrize("E,k", [(8, 1), (8, 8), (100, 7), (256, 8), (256, 32), (512, 22),
                                 (2560, 8), (2560, 22), (4096, 32), (33, 32)])
def test_route_shapes(cuda_dev, E, k):
    case = synth.make_case("tiny", device=cuda_dev, T=37, E=E, k=k, H=64)
    check_route(case)


@pytest.mark.parametrize("T,H,E,k,tp", [(37, 8192, 256, 8, 1), (64, 4096, 512, 22, 4), (19, 2048, 100, 7, 1),
                                        (40, 2688, 128, 8, 1), (16, 1024, 256, 8, 1),
                                        (24, 4096, 2560, 8, 4), (9, 16384, 512, 32, 1)])
def test_route_norm_quant_fused(cuda_dev, T, H, E, k, tp):
    """One launch (or the two kernels where the fused one does not apply) equals both stages."""
    case = synth.make_case("tiny", device=cuda_dev, T=T, H=H, E=E, k=k, tp=tp, join=False)
    ids, w, packed, sf = eb.moe_route_norm_quant(case.logits, case.bias, case.mask, case.k, case.x,
                                                 case.norm_w, case.gc, case.eps, case.gs, tp=tp)
    torch.cuda.synchronize()
    ids_o, w_o = oracle.route(synth.host(case.logits), synth.host(case.bias), synth.host(case.mask),
                              case.k)
    assert np.array_equal(synth.host(ids), ids_o)
    assert np.array_equal(synth.host(w).view(np.uint32), w_o.view(np.uint32))
    p_o, s_o = oracle.norm_quant(synth.host(case.x), case.T, case.H, tp, synth.host(case.norm_w),
                                 case.gc, case.eps, float(synth.host(case.gs)[0]))
    assert np.array_equal(synth.host(packed), p_o) and np.array_equal(synth.host(sf), s_o)
    assert eb.device_status() == 0


@pytest.mark.parametrize("T,H,E,k,tp,gc", [(889, 8192, 256, 8, 1, 0.0), (1500, 2048, 100, 7, 1, 1.0),
                                           (3001, 4096, 256, 8, 4, 0.0), (2000, 2688, 64, 8, 1, 1.0),
                                           (1200, 16384, 8, 1, 1, 0.0), (2048, 8192, 256, 32, 1, 1.0),
                                           (1000, 4096, 512, 8, 1, 0.0), (1300, 1024, 256, 8, 1, 1.0)])
def test_route_norm_quant_large_batches(cuda_dev, T, H, E, k, tp, gc):
    """Batches above the beside-router size: the router runs in extra warps of
    the wide norm-quant kernel (E <= 256, H >= 2048), else before it; either
    way both outputs equal the oracle's, masked tokens included."""
    case = synth.make_case("tiny", device=cuda_dev, T=T, H=H, E=E, k=k, tp=tp, gc=gc, join=False)
    assert (synth.host(case.mask) == 0).any()
    ids, w, packed, sf = eb.moe_route_norm_quant(case.logits, case.bias, case.mask, case.k, case.x,
                                                 case.norm_w, case.gc, case.eps, case.gs, tp=tp)
    torch.cuda.synchronize()
    ids_o, w_o = oracle.route(synth.host(case.logits), synth.host(case.bias), synth.host(case.mask),
                              case.k)
    assert np.array_equal(synth.host(ids), ids_o)
    assert np.array_equal(synth.host(w).view(np.uint32), w_o.view(np.uint32))
    p_o, s_o = oracle.norm_quant(synth.host(case.x), case.T, case.H, tp, synth.host(case.norm_w),
                                 case.gc, case.eps, float(synth.host(case.gs)[0]))
    assert np.array_equal(synth.host(packed), p_o) and np.array_equal(synth.host(sf), s_o)
    assert eb.device_status() == 0


def test_route_norm_quant_kernel_count(cuda_dev):
    sms = torch.cuda.get_device_properties(cuda_dev).multi_processor_count
    assert eb.route_norm_quant_kernels(8192, 8192, 256, 8) == 1
    assert eb.route_norm_quant_kernels(sms * 6 + 1, 2048, 100, 7) == 1
    assert eb.route_norm_quant_kernels(sms * 6, 8192, 256, 8) == 2       # router beside the norm-quant
    assert eb.route_norm_quant_kernels(8192, 8192, 512, 8) == 2          # router first
    assert eb.route_norm_quant_kernels(8192, 1024, 256, 8) == 2          # not the wide path


def test_route_integer_logits_many_ties(cuda_dev):
    g = torch.Generator(device=cuda_dev)
    g.manual_seed(5)
    for E, k in ((16, 5), (64, 8), (256, 8), (1024, 8), (2560, 22)):
        case = synth.make_case("tiny", device=cuda_dev, T=64, E=E, k=k, H=64)
        case.logits.copy_(torch.randint(-2, 3, case.logits.shape, generator=g, device=cuda_dev))
        vals = torch.tensor([0.0, 0.125, -0.125], device=cuda_dev)
        case.bias.copy_(vals[torch.randint(0, 3, (E,), generator=g, device=cuda_dev)])
        case.logits[case.mask == 0] = float("nan")
        check_route(case)


@pytest.mark.parametrize("H", [16, 48, 272, 1024, 2688, 4096, 8192, 16384])
@pytest.mark.parametrize("gc", [0.0, 1.0])
def test_norm_quant_hidden_sizes(cuda_dev, H, gc):
    case = synth.make_case("tiny", device=cuda_dev, T=19, H=H, gc=gc, join=False)
    check_norm_quant(case)


@pytest.mark.parametrize("H,tp", [(1024, 2), (1024, 4), (4096, 4), (4096, 8), (8192, 8), (768, 3)])
def test_norm_quant_rank_block(cuda_dev, H, tp):
    case = synth.make_case("tiny", device=cuda_dev, T=21, H=H, tp=tp, join=False)
    check_norm_quant(case)


def test_norm_quant_zero_scale_and_saturation(cuda_dev):
    case = synth.make_case("tiny", device=cuda_dev, T=8, H=256, join=False)
    x = case.x.float()
    x[0, :16] = 4.0                      # large block; the rest of row 0 tiny negatives
    x[0, 16:] = -1e-30
    x[1] = 0.0                           # an all-zero row: inv = 1/sqrt(eps)
    x[2, 32:48] = 1e4                    # one dominant block in row 2
    case.x.copy_(x.to(torch.bfloat16))
    case.gs.fill_(1e4)                   # large global scale: most block scales saturate at 448
    packed, sf, _ = check_norm_quant(case)
    s = synth.host(sf)
    assert (s[0, 1:] == 0).all() and (s == 0x7E).any()


@pytest.mark.parametrize("H,k", [(16, 1), (48, 3), (1024, 8), (1024, 22), (2688, 8), (4096, 8),
                                 (8192, 8), (16384, 4), (1024, 32)])
def test_combine_shapes(cuda_dev, H, k):
    case = synth.make_case("tiny", device=cuda_dev, T=23, H=H, k=k, E=max(64, k), join=False)
    check_combine(case)


@pytest.mark.parametrize("H", [1024, 2048, 2688, 8192, 16384])   # pair rows; wide rows of 1, 2 (partial), 4, 8 warps
def test_combine_gain_centre_one(cuda_dev, H):
    case = synth.make_case("tiny", device=cuda_dev, T=29, H=H, join=False)
    g = torch.Generator(device=cuda_dev)
    g.manual_seed(7)
    case.post_w.copy_((0.1 * torch.randn(H, generator=g, device=cuda_dev)).to(torch.bfloat16))
    case.post_gc = 1.0
    check_combine(case)


def test_combine_invalid_slots_never_read(cuda_dev):
    case = synth.make_case("tiny", device=cuda_dev)
    idx = case.row_idx
    assert (idx < 0).sum() >= 2 and (idx >= case.R).sum() == 1
    out, _ = check_combine(case)
    assert torch.isfinite(out.float()).all()
    # every slot invalid for one token: zeros, nothing read
    case.row_idx[4] = -1
    case.row_idx[6] = case.R + 1
    out, _ = check_combine(case)
    assert (out[4] == 0).all() and (out[6] == 0).all()


def test_combine_empty_and_no_rows(cuda_dev):
    case = synth.make_case("tiny", device=cuda_dev, T=4, H=64, k=2, E=8, join=False)
    case.row_idx.fill_(-1)
    out = eb.expert_combine(case.expert_out, 0, case.row_idx, case.comb_wt, case.post_w, 0.0, 1e-6)
    torch.cuda.synchronize()
    assert (out == 0).all()
    z = torch.empty(0, 2, dtype=torch.int32, device=cuda_dev)
    eb.expert_combine(case.expert_out, case.R, z, torch.empty(0, 2, device=cuda_dev),
                      case.post_w, 0.0, 1e-6)


@pytest.mark.parametrize("H", [64, 1024, 4096, 8192])
@pytest.mark.parametrize("with_next", [True, False])
def test_residual_join(cuda_dev, H, with_next):
    case = synth.make_case("tiny", device=cuda_dev, T=13, H=H, join=True)
    g = torch.Generator(device=cuda_dev)
    g.manual_seed(3)
    branch = torch.randn(case.T, H, generator=g, device=cuda_dev).to(torch.bfloat16)
    r = case.residual.clone()
    nw = case.next_w if with_next else None
    p = eb.residual_join(r, branch, case.gain, case.alpha, case.beta, case.eps, nw, case.next_gc,
                         case.eps)
    torch.cuda.synchronize()
    r_o, p_o, n_o = oracle.join(synth.host(case.residual), synth.host(branch), synth.host(case.gain),
                                case.alpha, case.beta, case.eps,
                                synth.host(nw) if with_next else None, case.next_gc, case.eps,
                                return_normed=True)
    check_join_outputs(synth.host(r), synth.host(p) if with_next else None, r_o, p_o, n_o, case.beta)


def test_combine_join_fused_equals_oracle_chain(cuda_dev):
    case = synth.make_case("tiny", device=cuda_dev, join=True)
    r = case.residual.clone()
    out, p = eb.expert_combine_join(case.expert_out, case.R, case.row_idx, case.comb_wt,
                                    case.post_w, case.post_gc, case.eps, r, case.gain, case.alpha,
                                    case.beta, case.eps, case.next_w, case.next_gc, case.eps,
                                    out=torch.empty(case.T, case.H, dtype=torch.bfloat16,
                                                    device=cuda_dev))
    torch.cuda.synchronize()
    branch_o = oracle_combine(case, synth.host(case.comb_wt))
    assert bf16_ulp_diff(synth.host(out), branch_o).max() <= 1
    r_o, p_o, n_o = oracle.join(synth.host(case.residual), branch_o, synth.host(case.gain), case.alpha,
                                case.beta, case.eps, synth.host(case.next_w), case.next_gc, case.eps,
                                return_normed=True)
    check_join_outputs(synth.host(r), synth.host(p), r_o, p_o, n_o, case.beta)


def test_route_then_combine_end_to_end(cuda_dev):
    """Stage 1's weights feed stage 3, on both sides."""
    case = synth.make_case("wide_topk", device=cuda_dev, T=300, join=False)
    ids, w = eb.moe_route(case.logits, case.bias, case.mask, case.k)
    torch.cuda.synchronize()
    _, w_o = oracle.route(synth.host(case.logits), synth.host(case.bias), synth.host(case.mask),
                          case.k)
    check_combine(case, wt=w, wt_host=w_o)


def test_nonblocking_stream_and_determinism(cuda_dev):
    case = synth.make_case("tiny", device=cuda_dev, T=64, H=2048, join=False)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        p1, s1 = eb.norm_quant_nvfp4(case.x, case.T, case.norm_w, 0.0, case.eps, case.gs)
        o1 = eb.expert_combine(case.expert_out, case.R, case.row_idx, case.comb_wt, case.post_w,
                               0.0, case.eps)
    s.synchronize()
    p2, s2 = eb.norm_quant_nvfp4(case.x, case.T, case.norm_w, 0.0, case.eps, case.gs)
    o2 = eb.expert_combine(case.expert_out, case.R, case.row_idx, case.comb_wt, case.post_w, 0.0,
                           case.eps)
    torch.cuda.synchronize()
    assert torch.equal(p1, p2) and torch.equal(s1, s2) and torch.equal(o1, o2)
    assert eb.device_status() == 0


def test_cuda_graph_replay_with_changed_inputs(cuda_dev):
    case = synth.make_case("tiny", device=cuda_dev, T=32, H=1024, join=False)
    ids = torch.empty(case.T, case.k, dtype=torch.int32, device=cuda_dev)
    w = torch.empty(case.T, case.k, dtype=torch.float32, device=cuda_dev)
    packed = torch.empty(case.T, case.H // 2, dtype=torch.uint8, device=cuda_dev)
    sf = torch.empty(case.T, case.H // 16, dtype=torch.uint8, device=cuda_dev)
    out = torch.empty(case.T, case.H, dtype=torch.bfloat16, device=cuda_dev)

    def step():
        eb.moe_route(case.logits, case.bias, case.mask, case.k, ids, w)
        eb.norm_quant_nvfp4(case.x, case.T, case.norm_w, 0.0, case.eps, case.gs, packed=packed,
                            sf=sf)
        eb.expert_combine(case.expert_out, case.R, case.row_idx, w, case.post_w, 0.0, case.eps,
                          out=out)

    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        step()                                  # warm-up (first call configures the kernels)
    torch.cuda.current_stream().wait_stream(s)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    for seed in (11, 12):
        other = synth.make_case("tiny", device=cuda_dev, T=32, H=1024, join=False, seed=seed)
        case.logits.copy_(other.logits)
        case.x.copy_(other.x)
        case.expert_buf.copy_(other.expert_buf)
        graph.replay()
        torch.cuda.synchronize()
        ids_o, w_o = oracle.route(synth.host(case.logits), synth.host(case.bias),
                                  synth.host(case.mask), case.k)
        assert np.array_equal(synth.host(ids), ids_o)
        p_o, s_o = oracle.norm_quant(synth.host(case.x), case.T, case.H, 1,
                                     synth.host(case.norm_w), 0.0, case.eps,
                                     float(synth.host(case.gs)[0]))
        assert np.array_equal(synth.host(packed), p_o) and np.array_equal(synth.host(sf), s_o)
        want = oracle_combine(case, w_o)
        assert bf16_ulp_diff(synth.host(out), want).max() <= 1


def test_invalid_arguments_raise(cuda_dev):
    case = synth.make_case("tiny", device=cuda_dev, T=4, H=64, k=2, E=8, join=False)
    with pytest.raises(eb.MoEBoundaryError) as ei:
        eb.moe_route(case.logits, case.bias, case.mask, 0)
    assert ei.value.status == 2
    with pytest.raises(eb.MoEBoundaryError):
        eb.norm_quant_nvfp4(case.x, case.T, case.norm_w, 0.0, 1e-6, case.gs, tp=3)
    bad = torch.empty(8 * 64 + 8, dtype=torch.bfloat16, device=cuda_dev)[1:][: 4 * 64]
    with pytest.raises(eb.MoEBoundaryError) as ei:
        eb.norm_quant_nvfp4(bad, 4, case.norm_w, 0.0, 1e-6, case.gs)
    assert ei.value.status == 1 and "aligned" in eb.last_error()


@pytest.mark.parametrize("T,H", [(100, 1024), (2000, 1024), (2000, 2048)])
def test_joint_pre_expert_steps_feed_the_combine(cuda_dev, T, H):
    """Several steps of (moe_route_norm_quant -> expert_combine) on one stream,
    new logits each step, no synchronisation in between: each step's combine
    must use that step's routing weights (the router running beside the
    norm-quant at 100 tokens, before it at 2000 x 1024, inside it at
    2000 x 2048)."""
    case = synth.make_case("tiny", device=cuda_dev, T=T, H=H, E=64, k=8, join=False)
    k, H = case.k, case.H
    ids = torch.empty(T, k, dtype=torch.int32, device=cuda_dev)
    w = torch.empty(T, k, dtype=torch.float32, device=cuda_dev)
    packed = torch.empty(T, H // 2, dtype=torch.uint8, device=cuda_dev)
    sf = torch.empty(T, H // 16, dtype=torch.uint8, device=cuda_dev)
    g = torch.Generator(device="cpu")
    g.manual_seed(17)
    logits_steps = [torch.randn(T, case.E, generator=g).to(cuda_dev) for _ in range(3)]
    outs = []
    for lg in logits_steps:
        case.logits.copy_(lg)
        eb.moe_route_norm_quant(case.logits, case.bias, case.mask, k, case.x, case.norm_w, case.gc,
                                case.eps, case.gs, topk_ids=ids, topk_weights=w, packed=packed, sf=sf)
        outs.append(eb.expert_combine(case.expert_out, case.R, case.row_idx, w, case.post_w, case.post_gc,
                                      case.eps))
    torch.cuda.synchronize()
    for lg, out in zip(logits_steps, outs):
        ids_o, w_o = oracle.route(synth.host(lg), synth.host(case.bias), synth.host(case.mask), k)
        assert bf16_ulp_diff(synth.host(out), oracle_combine(case, w_o)).max() <= 1
    assert eb.device_status() == 0


def test_fast_sigmoid_bound_holds_for_every_input(cuda_dev):
    """The router shortlists with a fast sigmoid and is exact only while that
    stays within its stated bound of the exact sigmoid: measured here over
    every binary32 input on this device."""
    err = eb.moe_route_check_fast_sigmoid()
    assert 0.0 < err <= eb.ROUTE_FAST_SIGMOID_BOUND, err


@pytest.mark.parametrize("E,k", [(256, 8), (512, 22), (64, 32), (33, 32), (2560, 8), (4096, 32), (1030, 9)])
def test_route_shortlist_overflow_takes_the_exact_rounds(cuda_dev, E, k):
    """Logits far above the sigmoid's saturation give many exactly equal
    scores, so more than 32 experts reach the shortlist window and the token
    takes the exact rounds; ties still go to the lowest ids."""
    case = synth.make_case("tiny", device=cuda_dev, T=40, E=E, k=k, H=64)
    case.logits[:20] = 40.0                    # every sigmoid rounds to 1: all scores tie on bias
    case.bias.zero_()
    case.logits[20:, : E // 2] = 40.0           # half the experts tie
    case.logits[case.mask == 0] = float("nan")
    ids, _, _ = check_route(case)
    got = synth.host(ids)
    assert (got[0] == np.arange(k)).all()


@pytest.mark.parametrize("E", [2560, 1024])
def test_route_large_e_lane_holding_many_candidates(cuda_dev, E):
    """Large E: experts 4, 8, 12 (one in each of lanes 1-3) score highest, and
    ten experts of lane 0's slice (0-3, 128-131, 256, 257) come next, so close
    together that all ten fall in the shortlist window -- more than one lane
    keeps -- and the token takes the exact rounds (their sigmoids partly tie,
    so the lowest ids win)."""
    k = 5
    case = synth.make_case("tiny", device=cuda_dev, T=8, E=E, k=k, H=64)
    lane0 = [0, 1, 2, 3, 128, 129, 130, 131, 256, 257]
    case.logits.fill_(-10.0)
    for n, e in enumerate(lane0):
        case.logits[:, e] = 5.0 + n * 1e-6
    for n, e in enumerate((4, 8, 12)):
        case.logits[:, e] = 6.0 + 0.1 * n
    case.bias.zero_()
    case.logits[case.mask == 0] = float("nan")
    ids, _, _ = check_route(case)
    got = synth.host(ids)[0].tolist()
    assert got[:3] == [12, 8, 4] and set(got[3:]) <= set(lane0)
