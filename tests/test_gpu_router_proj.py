"""Router projection on the tensor cores (tcgen05, BF16 operands with the FP32
weight prepared into three BF16 parts, FP32 accumulation) against the binary64
oracle.

Floating point with a documented bound: |got - exact| <= (2^-27 +
(3 H / C / 16 + 12) 2^-23) * sum |scale x w|, C the K chunks per expert tile.
Integer-valued inputs whose every partial sum is exact in FP32 must come out
exact; the prepared parts are compared bit for bit with the oracle's BF16
rounding.
"""
import numpy as np
import pytest
import torch

import expert_combine_b200 as eb
import oracle
from expert_combine_b200 import synth

pytestmark = pytest.mark.gpu


def _chunks(H):
    for c in (8, 4, 2):
        if H % (64 * c) == 0:
            return c
    return 1


def _logits(x, w, scale, dev):
    w3 = eb.router_weight_prepare(w.to(dev))
    return eb.router_logits(x.to(dev), w3, scale)


def _inputs(T, H, E, seed):
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    x = torch.randn(T, H, generator=g).to(torch.bfloat16)
    w = (torch.randn(E, H, generator=g) / H ** 0.5).to(torch.float32)
    return x, w


def _check(x, w, scale, dev):
    T, H = x.shape
    E = w.shape[0]
    got = _logits(x, w, scale, dev)
    torch.cuda.synchronize()
    ref, mag = oracle.router_logits(synth.host(x), w.numpy(), scale)
    err = np.abs(synth.host(got).astype(np.float64) - ref)
    bound = (2.0 ** -27 + (3 * H / _chunks(H) / 16 + 12) * 2.0 ** -23) * mag + 1e-30
    assert np.all(err <= bound), f"max err / bound {np.max(err / bound)}"
    return err, mag, got


@pytest.mark.parametrize("T,H,E", [(1, 1024, 256), (16, 8192, 256), (128, 8192, 256), (100, 4096, 2560),
                                   (37, 2688, 64), (200, 1024, 512), (5, 64, 16), (130, 192, 16),
                                   (64, 16384, 48)])
def test_router_logits_within_bound(cuda_dev, T, H, E):
    x, w = _inputs(T, H, E, seed=T * 7 + H)
    err, mag, _ = _check(x, w, 0.37, cuda_dev)
    # typical error far below the worst-case bound: FP32-level
    assert np.median(err / mag) < 2e-7


def test_router_logits_exact_on_small_integers(cuda_dev):
    # |x| <= 16 and |w| <= 255 are exact in BF16 / TF32, every product and
    # partial sum is an integer below 2^24 (2048 * 16 * 255 < 2^23): the
    # result is exact in any order
    g = torch.Generator(device="cpu")
    g.manual_seed(3)
    T, H, E = 96, 2048, 32
    x = torch.randint(-16, 17, (T, H), generator=g).to(torch.bfloat16)
    w = torch.randint(-255, 256, (E, H), generator=g).to(torch.float32)
    got = _logits(x, w, 1.0, cuda_dev)
    torch.cuda.synchronize()
    want = x.to(torch.int64) @ w.to(torch.int64).T
    assert np.array_equal(synth.host(got).astype(np.int64), want.numpy())


def test_router_logits_weight_remainder_matters(cuda_dev):
    """Weights with bits below BF16 precision: a product on the first part
    alone would miss them by up to 2^-9 relative; the other two parts keep
    the result at FP32 level."""
    T, H, E = 32, 1024, 16
    x, w = _inputs(T, H, E, seed=11)
    w = w + w * (2.0 ** -12)             # fill the low mantissa bits
    err, mag, _ = _check(x, w, 1.0, cuda_dev)
    assert np.max(err / mag) < 2.0 ** -18


def test_router_logits_reproducible_and_zero_tokens(cuda_dev):
    x, w = _inputs(77, 8192, 256, seed=5)
    w3 = eb.router_weight_prepare(w.to(cuda_dev))
    a = eb.router_logits(x.to(cuda_dev), w3, 1.0)
    b = eb.router_logits(x.to(cuda_dev), w3, 1.0)
    torch.cuda.synchronize()
    assert torch.equal(a, b)
    z = eb.router_logits(torch.empty(0, 8192, dtype=torch.bfloat16, device=cuda_dev), w3, 1.0)
    assert z.shape == (0, 256)
    assert eb.device_status() == 0


def test_router_logits_feed_the_router(cuda_dev):
    """Projection -> routing on the GPU: the router's picks equal the oracle's
    routing of the projected logits (the router's input taken as given)."""
    T, H, E, k = 128, 8192, 256, 8
    x, w = _inputs(T, H, E, seed=21)
    logits = _logits(x, w, 1.0, cuda_dev)
    bias = torch.zeros(E, dtype=torch.float32, device=cuda_dev)
    mask = torch.ones(T, dtype=torch.uint8, device=cuda_dev)
    ids, wts = eb.moe_route(logits, bias, mask, k)
    torch.cuda.synchronize()
    ids_o, _ = oracle.route(synth.host(logits), synth.host(bias), synth.host(mask), k)
    assert np.array_equal(synth.host(ids), ids_o)


def test_router_weight_prepare_parts(cuda_dev):
    """The three BF16 parts: each the round-to-nearest-even of the remainder
    left by the previous ones (the oracle's BF16 rounding, NumPy's FP32
    subtraction), and their sum within 2^-27 of the weight."""
    g = torch.Generator(device="cpu")
    g.manual_seed(13)
    E, H = 48, 1024
    w = torch.randn(E, H, generator=g) * torch.exp(4 * torch.randn(E, H, generator=g))
    w3 = eb.router_weight_prepare(w.to(cuda_dev))
    torch.cuda.synchronize()
    got = synth.host(w3)
    wn = w.numpy()
    b1 = oracle.bf16_rn_array(wn)
    r1 = (wn - (b1.astype(np.uint32) << 16).view(np.float32)).astype(np.float32)
    b2 = oracle.bf16_rn_array(r1)
    r2 = (r1 - (b2.astype(np.uint32) << 16).view(np.float32)).astype(np.float32)
    b3 = oracle.bf16_rn_array(r2)
    assert np.array_equal(got[0], b1) and np.array_equal(got[1], b2) and np.array_equal(got[2], b3)
    parts = sum(((got[p].astype(np.uint32) << 16).view(np.float32).astype(np.float64)) for p in range(3))
    assert np.all(np.abs(parts - wn.astype(np.float64)) <= 2.0 ** -27 * np.abs(wn.astype(np.float64)))


def _experts_per_cta(T, E, H, sms):
    """The tile the launch picks: 32 experts per CTA when E allows it and the
    16-expert grid would take more than one wave at two CTAs per SM."""
    ctas16 = (E // 16) * _chunks(H) * ((T + 127) // 128)
    return 32 if E % 32 == 0 and ctas16 > 2 * sms else 16


@pytest.mark.parametrize("T_small,T_big,H,E", [(128, 512, 8192, 256),     # C = 8
                                               (100, 700, 64, 1024),      # C = 1, partial last tile
                                               (60, 300, 128, 1024),      # C = 2
                                               (90, 300, 256, 512)])      # C = 4
def test_router_logits_equal_across_tile_widths(cuda_dev, T_small, T_big, H, E):
    """The rows a small batch shares with a larger one come out bit-identical
    whether the launch takes 16 or 32 experts per CTA (every output element is
    summed in the same order either way)."""
    sms = torch.cuda.get_device_properties(cuda_dev).multi_processor_count
    assert _experts_per_cta(T_small, E, H, sms) == 16 and _experts_per_cta(T_big, E, H, sms) == 32
    x, w = _inputs(T_big, H, E, seed=T_big + H + E)
    w3 = eb.router_weight_prepare(w.to(cuda_dev))
    xd = x.to(cuda_dev)
    small = eb.router_logits(xd[:T_small].contiguous(), w3, 0.37)
    big = eb.router_logits(xd, w3, 0.37)
    torch.cuda.synchronize()
    assert torch.equal(small, big[:T_small])
    _check(x, w, 0.37, cuda_dev)
