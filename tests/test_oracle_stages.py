"""Pins of the oracle's three stages and the join (CPU only).

Pins come from outside the oracle: a hand-worked golden example, brute-force
selection with Python's sort, float64 evaluation of the defining formulas
within their rounding bounds, closed forms and invariants (layout equivalence,
permutation invariance, NaN never read, identities of the join).
"""
import os

import numpy as np
import pytest
import torch

import oracle
from expert_combine_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def bf16_bits(a):
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(torch.bfloat16) \
        .view(torch.int16).numpy().view(np.uint16)


def bits_to_f32(u16):
    return (np.asarray(u16, np.uint16).astype(np.uint32) << 16).view(np.float32)


def bf16_ulp(v):
    """Spacing of BF16 numbers at |v| (float64)."""
    v = np.maximum(np.abs(np.asarray(v, np.float64)), 2.0 ** -126)
    return 2.0 ** (np.floor(np.log2(v)) - 7)


# ======================================================================
# stage 1: router
# ======================================================================
def test_route_golden_worked_example():
    kv = {}
    with open(os.path.join(GOLDEN, "route_worked.txt")) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                key, *vals = line.split()
                kv[key] = vals
    E, k = int(kv["E"][0]), int(kv["k"][0])
    logits = np.array(kv["logits"], np.float32).reshape(1, E)
    bias = np.array(kv["bias"], np.float32)
    ids, w = oracle.route(logits, bias, np.ones(1, np.uint8), k)
    assert ids[0].tolist() == [int(v) for v in kv["ids"]]
    assert [f"{u:08x}" for u in w[0].view(np.uint32)] == kv["weights_hex"]


def _brute_route(logits, bias, mask, k):
    T, E = logits.shape
    ids = np.full((T, k), -1, np.int32)
    w = np.zeros((T, k), np.float32)
    s_all = oracle.sigmoid_array(logits)
    for t in range(T):
        if not mask[t]:
            continue
        s = s_all[t]
        c = (s + bias).astype(np.float32)
        order = sorted(range(E), key=lambda e: (-float(c[e]), e))[:k]
        S = np.float32(0)
        for e in order:
            S = np.float32(S + s[e])
        ids[t] = order
        w[t] = [np.float32(s[e] / S) for e in order]
    return ids, w


def test_route_brute_force_tiny_with_many_ties():
    rng = np.random.default_rng(2024)
    for E in (4, 8, 16):
        for k in range(1, E + 1):
            T = 12
            logits = rng.integers(-2, 3, (T, E)).astype(np.float32)
            bias = rng.choice(np.array([0.0, 0.125, -0.125], np.float32), E)
            mask = (rng.random(T) > 0.2).astype(np.uint8)
            logits[mask == 0] = np.nan
            got = oracle.route(logits, bias, mask, k)
            want = _brute_route(logits, bias, mask, k)
            assert np.array_equal(got[0], want[0]), (E, k)
            assert np.array_equal(got[1].view(np.uint32), want[1].view(np.uint32)), (E, k)


def test_route_zero_bias_distinct_logits_is_argsort():
    rng = np.random.default_rng(9)
    for E, k in ((256, 8), (512, 22), (2560, 8)):
        T = 8
        base = np.linspace(-3.0, 3.0, E, dtype=np.float32)
        logits = np.stack([rng.permutation(base) for _ in range(T)])
        ids, w = oracle.route(logits, np.zeros(E, np.float32), np.ones(T, np.uint8), k)
        want = np.argsort(-logits, axis=1, kind="stable")[:, :k]
        assert np.array_equal(ids, want)
        # weights are descending with the logits and sum to one
        assert np.all(np.diff(w, axis=1) <= 0)


def test_route_weights_sum_to_one_and_masked_tokens_empty():
    case = synth.make_case("tiny")
    logits, bias, mask = (synth.host(case.logits), synth.host(case.bias), synth.host(case.mask))
    ids, w = oracle.route(logits, bias, mask, case.k)
    valid = mask.astype(bool)
    assert np.all(ids[~valid] == -1) and np.all(w[~valid] == 0)
    assert np.all(np.abs(w[valid].astype(np.float64).sum(1) - 1.0) <= 1e-6)
    assert np.all((ids[valid] >= 0) & (ids[valid] < case.E))
    for row in ids[valid]:
        assert len(set(row.tolist())) == case.k
    # the three injected exact ties (see synth.TIE_PAIRS)
    assert 10 in ids[0] and 11 not in ids[0] and ids[0][-1] == 10
    r1 = ids[1].tolist()
    assert 20 in r1 and 21 in r1 and r1.index(20) + 1 == r1.index(21)
    assert 30 not in ids[2] and 31 not in ids[2]


def test_route_against_full_numpy_sort_large_e():
    rng = np.random.default_rng(77)
    T, E, k = 24, 2560, 8
    logits = rng.standard_normal((T, E)).astype(np.float32)
    bias = rng.uniform(-0.05, 0.05, E).astype(np.float32)
    ids, w = oracle.route(logits, bias, np.ones(T, np.uint8), k)
    s = oracle.sigmoid_array(logits)
    c = (s + bias[None, :]).astype(np.float32)
    for t in range(T):
        order = np.lexsort((np.arange(E), -c[t].astype(np.float64)))[:k]
        assert np.array_equal(ids[t], order)


# ======================================================================
# stage 2: RMSNorm + NVFP4
# ======================================================================
def _exact_norm(xf, w_f, gc, eps):
    x64 = xf.astype(np.float64)
    inv = 1.0 / np.sqrt(np.mean(x64 ** 2, axis=-1, keepdims=True) + eps)
    return x64 * (gc + w_f.astype(np.float64)) * inv


@pytest.mark.parametrize("H,tp", [(1024, 1), (1024, 2), (4096, 4), (2688, 1), (48, 3)])
def test_norm_matches_float64_within_one_bf16_ulp(H, tp):
    rng = np.random.default_rng(H + tp)
    M = 9
    xl = bf16_bits(rng.standard_normal((M, H)))
    w = bf16_bits(rng.normal(1.0, 0.1, H))
    x = xl if tp == 1 else np.ascontiguousarray(xl.reshape(M, tp, H // tp).transpose(1, 0, 2))
    y = oracle.norm_bf16(x, M, H, tp, w, 0.0, 1e-6)
    ref = _exact_norm(bits_to_f32(xl), bits_to_f32(w), 0.0, 1e-6)
    err = np.abs(bits_to_f32(y).astype(np.float64) - ref)
    assert np.all(err <= bf16_ulp(ref) * 0.5 + np.abs(ref) * 2.0 ** -20)


def test_rank_block_layout_equals_contiguous():
    rng = np.random.default_rng(1)
    M, H = 7, 1024
    xl = bf16_bits(rng.standard_normal((M, H)))
    w = bf16_bits(rng.normal(1.0, 0.1, H))
    gs = np.float32(2688.0) / np.float32(np.abs(bits_to_f32(xl)).max())
    p1, s1 = oracle.norm_quant(xl, M, H, 1, w, 0.0, 1e-6, gs)
    for tp in (2, 4, 8):
        xr = np.ascontiguousarray(xl.reshape(M, tp, H // tp).transpose(1, 0, 2))
        p, s = oracle.norm_quant(xr, M, H, tp, w, 0.0, 1e-6, gs)
        assert np.array_equal(p, p1) and np.array_equal(s, s1)


def test_gain_centre_adds_one_in_fp32():
    rng = np.random.default_rng(4)
    M, H = 5, 256
    xl = bf16_bits(rng.standard_normal((M, H)))
    # offsets that are multiples of 2^-7 in [-0.5, 0.5]: 1 + w is exact in BF16
    off = (rng.integers(-64, 65, H) / 128.0).astype(np.float32)
    y1 = oracle.norm_bf16(xl, M, H, 1, bf16_bits(off), 1.0, 1e-6)
    y0 = oracle.norm_bf16(xl, M, H, 1, bf16_bits(off + 1.0), 0.0, 1e-6)
    assert np.array_equal(y0, y1)


def _decode_codes(packed):
    lo = packed & 0x0F
    hi = packed >> 4
    codes = np.stack([lo, hi], axis=-1).reshape(packed.shape[0], -1)
    grid = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
    val = grid[codes & 7]
    return np.where(codes & 8, -val, val), codes


@pytest.mark.parametrize("gc", [0.0, 1.0])
def test_norm_quant_codes_and_scales_against_independent_quantiser(gc):
    case = synth.make_case("tiny", T=16, H=1024, gc=gc)
    M, H = case.T, case.H
    x, w = synth.host(case.x), synth.host(case.norm_w)
    gs = np.float32(synth.host(case.gs)[0])
    packed, sf = oracle.norm_quant(x, M, H, 1, w, gc, case.eps, gs)
    y = bits_to_f32(oracle.norm_bf16(x, M, H, 1, w, gc, case.eps)).reshape(M, H // 16, 16)
    # scale: library E4M3 cast of the saturated product gs * (amax * fl(1/6))
    amax = np.abs(y).max(-1)
    u = (gs * (amax * np.float32(1.0 / 6.0)).astype(np.float32)).astype(np.float32)
    sf_lib = torch.from_numpy(np.clip(u, -448, 448)).to(torch.float8_e4m3fn)
    assert np.array_equal(sf, sf_lib.view(torch.uint8).numpy())
    sf_f = sf_lib.float().numpy()
    with np.errstate(divide="ignore"):
        os_ = np.where(sf_f != 0, np.float32(1.0) / (sf_f * (np.float32(1.0) / gs)), 0.0)
    q = (y * os_.astype(np.float32)[..., None]).astype(np.float32)
    # codes: nearest grid point with ties to even, by exhaustive search
    grid = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
    m = np.minimum(np.abs(q.astype(np.float64)), 7.0)
    d = np.abs(m[..., None] - grid)
    near = d == d.min(-1, keepdims=True)
    code = np.argmin(np.where(near, np.arange(8) & 1, 2), -1).astype(np.uint8)
    code[q < 0] |= 8
    _, got = _decode_codes(packed)
    assert np.array_equal(got.reshape(M, H // 16, 16), code)


def test_norm_quant_invariants():
    case = synth.make_case("tiny", T=16, H=1024)
    M, H = case.T, case.H
    x, w = synth.host(case.x), synth.host(case.norm_w)
    gs = np.float32(synth.host(case.gs)[0])
    packed, sf = oracle.norm_quant(x, M, H, 1, w, 0.0, case.eps, gs)
    y = bits_to_f32(oracle.norm_bf16(x, M, H, 1, w, 0.0, case.eps)).astype(np.float64)
    dq, codes = _decode_codes(packed)
    sf_f = torch.from_numpy(sf).view(torch.float8_e4m3fn).float().numpy().astype(np.float64)
    assert np.all(sf <= 0x7E)                                # never NaN, at most 448
    assert np.abs(dq).max() <= 6.0
    scale = np.repeat(sf_f, 16, axis=1) / float(gs)
    rec = dq * scale
    q = np.abs(y) / np.where(scale > 0, scale, np.inf)
    half_step = np.where(q < 2, 0.25, np.where(q < 4, 0.5, 1.0))
    ok = (np.abs(rec - y) <= half_step * scale * (1 + 1e-6) + 1e-30) | (q > 6)
    assert ok.all()
    # the block(s) holding the tensor's largest input magnitude saturate the scale
    assert (sf == 0x7E).any()


def test_norm_quant_zero_scale_blocks_give_zero_codes():
    M, H = 2, 64
    xf = np.zeros((M, H), np.float32)
    xf[:, :16] = 1.0                      # block 0 large, blocks 1..3 tiny negatives
    xf[:, 16:] = -1e-30
    x = bf16_bits(xf)
    w = bf16_bits(np.ones(H))
    packed, sf = oracle.norm_quant(x, M, H, 1, w, 0.0, 1e-6, np.float32(1.0))
    assert np.all(sf[:, 1:] == 0)
    _, codes = _decode_codes(packed)
    # scale 0 -> q = y * 0 = -0.0: no sign bit under the pages' "scaled < 0" rule
    assert np.all(codes[:, 16:] == 0)


# ======================================================================
# stage 3: combine
# ======================================================================
def _exact_combine(expert, R, idx, wt, w, gc, eps):
    T, k = idx.shape
    out = np.zeros((T, expert.shape[1]))
    for t in range(T):
        for j in range(k):
            r = idx[t, j]
            if 0 <= r < R:
                out[t] += wt[t, j] * _exact_norm(bits_to_f32(expert[r]), bits_to_f32(w), gc, eps)
    return out


def test_combine_single_slot_is_the_norm():
    rng = np.random.default_rng(12)
    R, H, T = 10, 512, 10
    expert = bf16_bits(rng.standard_normal((R, H)))
    w = bf16_bits(rng.normal(1, 0.1, H))
    idx = rng.permutation(R).astype(np.int32).reshape(T, 1)
    out = oracle.combine(expert, R, idx, np.ones((T, 1), np.float32), w, 0.0, 1e-6)
    y = oracle.norm_bf16(expert, R, H, 1, w, 0.0, 1e-6)
    assert np.array_equal(out, y[idx[:, 0]])


def test_combine_never_reads_invalid_rows_and_matches_float64():
    case = synth.make_case("tiny")
    buf = synth.host(case.expert_buf)
    G, R = case.guard, case.R
    idx = synth.host(case.row_idx)
    wt = synth.host(case.comb_wt)
    w = synth.host(case.post_w)
    # the oracle receives the rows from R on (NaN guards) as readable memory
    out = oracle.combine(buf[G:], R, idx, wt, w, case.post_gc, case.eps)
    outf = bits_to_f32(out).astype(np.float64)
    assert np.isfinite(outf).all()
    assert (idx < 0).sum() >= 2 and (idx >= R).sum() == 1
    ref = _exact_combine(buf[G:], R, idx, wt, w, case.post_gc, case.eps)
    # each slot's BF16 norm is within half a BF16 step, the sum adds one rounding
    bound = np.zeros_like(ref)
    for t in range(case.T):
        for j in range(case.k):
            r = idx[t, j]
            if 0 <= r < R:
                yj = _exact_norm(bits_to_f32(buf[G + r]), bits_to_f32(w), 0.0, case.eps)
                bound[t] += wt[t, j] * (bf16_ulp(yj) * 0.5 + np.abs(yj) * 2.0 ** -20)
    bound += bf16_ulp(ref) * 0.5 + 1e-30
    assert np.all(np.abs(outf - ref) <= bound)
    masked = synth.host(case.mask) == 0
    assert np.all(out[masked] == 0)


def test_combine_row_permutation_invariance():
    rng = np.random.default_rng(13)
    R, H, T, k = 40, 256, 8, 5
    expert = bf16_bits(rng.standard_normal((R, H)))
    idx = rng.choice(R, (T, k), replace=False).astype(np.int32)
    wt = rng.random((T, k)).astype(np.float32)
    w = bf16_bits(rng.normal(1, 0.1, H))
    out = oracle.combine(expert, R, idx, wt, w, 0.0, 1e-6)
    perm = rng.permutation(R)
    inv = np.argsort(perm)
    out2 = oracle.combine(expert[perm], R, inv[idx].astype(np.int32), wt, w, 0.0, 1e-6)
    assert np.array_equal(out, out2)


def test_combine_all_invalid_token_is_zero():
    H = 64
    expert = np.full((4, H), 0x7FC0, np.uint16)             # NaN everywhere
    idx = np.array([[-1, 4, 7, -5]], np.int32)
    out = oracle.combine(expert, 4, idx, np.ones((1, 4), np.float32),
                         bf16_bits(np.ones(H)), 0.0, 1e-6)
    assert np.all(out == 0)


# ======================================================================
# gated residual join
# ======================================================================
def test_join_identities():
    rng = np.random.default_rng(21)
    T, H = 4, 512
    r = rng.standard_normal((T, H)).astype(np.float32)
    branch = bf16_bits(rng.standard_normal((T, H)))
    gain = bf16_bits(rng.normal(1, 0.1, H))
    r1, _ = oracle.join(r, branch, gain, 1.0, 0.0, 1e-6)
    assert np.array_equal(r1, r)
    r2, _ = oracle.join(r, np.zeros((T, H), np.uint16), gain, 0.75, 0.5, 1e-6)
    assert np.array_equal(r2, (np.float32(0.75) * r).astype(np.float32))


def test_join_and_prenorm_match_float64():
    case = synth.make_case("tiny", join=True)
    T, H = case.T, case.H
    rng = np.random.default_rng(8)
    branch = bf16_bits(rng.standard_normal((T, H)))
    r0 = synth.host(case.residual)
    gain, nw = synth.host(case.gain), synth.host(case.next_w)
    r1, p = oracle.join(r0, branch, gain, case.alpha, case.beta, case.eps, nw, case.next_gc,
                        case.eps)
    g = bits_to_f32(branch).astype(np.float64) * bits_to_f32(gain)
    n = g / np.sqrt(np.mean(g ** 2, -1, keepdims=True) + case.eps)
    ref = case.alpha * r0.astype(np.float64) + case.beta * n
    tol = case.beta * (bf16_ulp(n) * 1.5 + np.abs(n) * 2.0 ** -8) + np.abs(ref) * 1e-6
    assert np.all(np.abs(r1 - ref) <= tol)
    pref = _exact_norm(r1, bits_to_f32(nw), case.next_gc, case.eps)
    err = np.abs(bits_to_f32(p).astype(np.float64) - pref)
    assert np.all(err <= bf16_ulp(pref) * 0.5 + np.abs(pref) * 2.0 ** -20)
