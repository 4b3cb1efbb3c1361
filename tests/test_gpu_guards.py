"""Every entry point writes inside its outputs and nowhere else: each output
is the middle of a larger buffer whose 4 KiB before and after are filled with
a byte pattern, and the pattern must survive the call (an out-of-bounds-write
check that stands in for a memory sanitizer).  Shapes include ragged tails
and each arrangement of the router and the norm-quant."""
import numpy as np
import pytest
import torch

import expert_combine_b200 as eb
from expert_combine_b200 import synth

pytestmark = pytest.mark.gpu

G = 4096
PAT = 0x5A


class Guarded:
    def __init__(self, shape, dtype, dev):
        n = int(np.prod(shape)) * torch.empty(0, dtype=dtype).element_size()
        self.n = n
        self.buf = torch.full((G + n + G,), PAT, dtype=torch.uint8, device=dev)
        self.t = self.buf[G:G + n].view(dtype).view(shape)

    def intact(self):
        b = self.buf.cpu().numpy()
        return bool((b[:G] == PAT).all() and (b[G + self.n:] == PAT).all())


def _check(*gs):
    torch.cuda.synchronize()
    for g in gs:
        assert g.intact(), "a kernel wrote outside its output"


@pytest.mark.parametrize("T,H,E,k", [(37, 1040, 100, 7), (1500, 2048, 64, 8), (200, 8192, 256, 8),
                                     (1000, 4096, 512, 22)])
def test_pre_expert_outputs(cuda_dev, T, H, E, k):
    case = synth.make_case("tiny", device=cuda_dev, T=T, H=H, E=E, k=k, join=False)
    ids, w = Guarded((T, k), torch.int32, cuda_dev), Guarded((T, k), torch.float32, cuda_dev)
    packed, sf = Guarded((T, H // 2), torch.uint8, cuda_dev), Guarded((T, H // 16), torch.uint8, cuda_dev)
    eb.moe_route_norm_quant(case.logits, case.bias, case.mask, k, case.x, case.norm_w, case.gc, case.eps,
                            case.gs, topk_ids=ids.t, topk_weights=w.t, packed=packed.t, sf=sf.t)
    _check(ids, w, packed, sf)
    eb.moe_route(case.logits, case.bias, case.mask, k, ids.t, w.t)
    eb.norm_quant_nvfp4(case.x, T, case.norm_w, case.gc, case.eps, case.gs, packed=packed.t, sf=sf.t)
    _check(ids, w, packed, sf)


@pytest.mark.parametrize("T,H,k", [(3, 16, 1), (37, 1040, 7), (128, 8192, 8), (700, 4096, 8)])
def test_combine_and_join_outputs(cuda_dev, T, H, k):
    case = synth.make_case("tiny", device=cuda_dev, T=T, H=H, k=k, E=max(k, 64), join=True)
    out = Guarded((T, H), torch.bfloat16, cuda_dev)
    eb.expert_combine(case.expert_out, case.R, case.row_idx, case.comb_wt, case.post_w, case.post_gc, case.eps,
                      out=out.t)
    _check(out)
    res = Guarded((T, H), torch.float32, cuda_dev)
    res.t.copy_(case.residual)
    nxt = Guarded((T, H), torch.bfloat16, cuda_dev)
    eb.expert_combine_join(case.expert_out, case.R, case.row_idx, case.comb_wt, case.post_w, case.post_gc,
                           case.eps, res.t, case.gain, case.alpha, case.beta, case.eps, case.next_w, case.next_gc,
                           case.eps, out=out.t, next_prenorm=nxt.t)
    _check(out, res, nxt)
    eb.residual_join(res.t, out.t, case.gain, case.alpha, case.beta, case.eps, case.next_w, case.next_gc,
                     case.eps, next_prenorm=nxt.t)
    _check(res, nxt)


@pytest.mark.parametrize("T,k,E", [(5, 3, 16), (128, 8, 256), (3000, 8, 256), (4000, 22, 512)])
def test_dispatch_outputs(cuda_dev, T, k, E):
    ids = synth.make_topk_ids(T, k, E, seed=T, device=cuda_dev)
    off, idx, tok = (Guarded((E + 1,), torch.int32, cuda_dev), Guarded((T, k), torch.int32, cuda_dev),
                     Guarded((T * k,), torch.int32, cuda_dev))
    eb.moe_dispatch(ids, E, 0, off.t, idx.t, tok.t)
    _check(off, idx, tok)


def test_router_logits_and_finalize_outputs(cuda_dev):
    g = torch.Generator(device="cpu")
    g.manual_seed(2)
    x = torch.randn(100, 4096, generator=g).to(torch.bfloat16).to(cuda_dev)
    w = (torch.randn(48, 4096, generator=g) / 64).to(cuda_dev)
    w3 = Guarded((3, 48, 4096), torch.bfloat16, cuda_dev)
    eb.router_weight_prepare(w, w3=w3.t)
    lg = Guarded((100, 48), torch.float32, cuda_dev)
    eb.router_logits(x, w3.t, 1.0, logits=lg.t)
    _check(w3, lg)

    c = synth.make_ep_case(37, 1040, 8, 64, 3, seed=4, device=cuda_dev)
    n = eb.finalize_ar_workspace_size(3, 40, 1040)
    ws = [Guarded((n,), torch.uint8, cuda_dev) for _ in range(3)]
    for wg in ws:
        eb.finalize_ar_workspace_init(wg.t, 3, 40, 1040)
    outs = [Guarded((37, 1040), torch.bfloat16, cuda_dev) for _ in range(3)]
    eb.expert_finalize_allreduce_local(c.expert_out, c.R, c.row_idx, [c.weights] * 3, c.norm_w, c.gc, c.eps,
                                       [wg.t for wg in ws], 40, outs=[o.t for o in outs])
    _check(*ws, *outs)
    assert eb.device_status() == 0
