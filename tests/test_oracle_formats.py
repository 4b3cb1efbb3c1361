"""Pins of the oracle's number formats and scalar helpers (CPU only).

Each pin checks the oracle against something other than itself: the values
printed on the pages (E2M1 grid), a library implementation of the format
(torch's bfloat16 and float8_e4m3fn), a brute-force nearest search, libm's exp
in float64, or hand-derived binary32 results.
"""
import os

import numpy as np
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def _read_pairs(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(line.split())
    return rows


# ---------------------------------------------------------------- E2M1
def test_e2m1_printed_grid_and_ties():
    rows = _read_pairs("e2m1_grid.txt")
    assert len(rows) >= 20
    for q, code in rows:
        assert oracle.e2m1_code(float(q)) == int(code), q


def _brute_e2m1(q):
    """Nearest grid point by exhaustive distance, ties to the even code."""
    # beyond the largest grid point every magnitude is nearest to 6; clipping
    # keeps the float64 distances exact
    m = np.minimum(np.abs(q.astype(np.float64)), 7.0)
    d = np.abs(m[:, None] - GRID[None, :])
    nearest = d == d.min(axis=1, keepdims=True)
    # among the nearest grid points prefer the even code (round half to even)
    score = np.where(nearest, (np.arange(8) & 1)[None, :], 2)
    code = np.argmin(score, axis=1).astype(np.uint8)
    code[q < 0] |= 8
    return code


def _threshold_neighbourhood():
    pts = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, *GRID, 6.0], np.float32)
    out = [pts]
    for direction in (np.inf, -np.inf):
        cur = pts.copy()
        for _ in range(64):
            cur = np.nextafter(cur, np.float32(direction))
            out.append(cur.copy())
    v = np.concatenate(out)
    return np.concatenate([v, -v])


def test_e2m1_threshold_rule_equals_nearest_even_search():
    bits = np.arange(0, 2 ** 32, 4099, dtype=np.uint64).astype(np.uint32)
    q = bits.view(np.float32)
    q = q[np.isfinite(q)]
    q = np.concatenate([q, _threshold_neighbourhood(), np.array([np.inf, -np.inf], np.float32)])
    got = oracle.e2m1_code_array(q)
    want = _brute_e2m1(q)
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, (q[bad[:5]], got[bad[:5]], want[bad[:5]])


# ---------------------------------------------------------------- E4M3
def test_e4m3_decode_matches_library_format():
    codes = torch.arange(256, dtype=torch.uint8)
    lib = codes.view(torch.float8_e4m3fn).float().numpy()
    ours = np.array([oracle.e4m3_decode(c) for c in range(256)], np.float32)
    nan = np.isnan(lib)
    assert np.array_equal(nan, np.isnan(ours)) and nan.sum() == 2      # 0x7f and 0xff
    assert np.array_equal(lib[~nan], ours[~nan])
    assert ours[0x7E] == 448.0 and ours[1] == 2.0 ** -9


def test_e4m3_rounding_matches_library_cast_with_saturation():
    rng = np.random.default_rng(7)
    vals = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).float().numpy()
    fin = np.sort(vals[np.isfinite(vals) & (vals >= 0)])
    mids = ((fin[1:].astype(np.float64) + fin[:-1]) / 2).astype(np.float32)
    near = [mids]
    for direction in (np.inf, -np.inf):
        cur = mids.copy()
        for _ in range(3):
            cur = np.nextafter(cur, np.float32(direction))
            near.append(cur.copy())
    x = np.concatenate([
        (rng.standard_normal(300_000) * 60).astype(np.float32),
        np.ldexp(rng.random(100_000), -9).astype(np.float32),
        *near, fin, np.array([448.0, 449.0, 463.9, 464.0, 465.0, 1e9, np.inf], np.float32),
    ])
    x = np.concatenate([x, -x])
    ours = oracle.e4m3_rn_sat_array(x)
    lib = torch.from_numpy(np.clip(x, -448.0, 448.0)).to(torch.float8_e4m3fn)
    lib = lib.view(torch.uint8).numpy()
    bad = np.nonzero(ours != lib)[0]
    assert bad.size == 0, (x[bad[:5]], ours[bad[:5]], lib[bad[:5]])
    assert oracle.e4m3_rn_sat(1e30) == 0x7E                  # saturates, never NaN


# ---------------------------------------------------------------- BF16
def test_bf16_rounding_matches_library_cast():
    rng = np.random.default_rng(3)
    x = np.concatenate([
        rng.standard_normal(200_000).astype(np.float32),
        (rng.standard_normal(50_000) * 1e30).astype(np.float32),
        np.ldexp(rng.random(50_000), -130).astype(np.float32),
        rng.integers(0, 2 ** 32, 200_000, dtype=np.uint64).astype(np.uint32).view(np.float32),
    ])
    x = x[np.isfinite(x)]
    # exact halfway cases: low 16 bits 0x8000 with both parities of bit 16
    hw = (rng.integers(0, 2 ** 15, 1000, dtype=np.uint32) << 17 | 0x8000).view(np.float32)
    hw2 = (rng.integers(0, 2 ** 15, 1000, dtype=np.uint32) << 17 | 0x18000).view(np.float32)
    x = np.concatenate([x, hw, hw2])
    x = x[np.isfinite(x)]
    ours = oracle.bf16_rn_array(x)
    lib = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, lib)


# ---------------------------------------------------------------- exp / sigmoid
def _ulp_diff(a, b):
    ia = a.view(np.int32).astype(np.int64)
    ib = b.view(np.int32).astype(np.int64)
    return np.abs(ia - ib)


def test_exp_within_two_ulp_of_libm():
    x = np.linspace(-86.9, 87.9, 2_000_003, dtype=np.float32)
    ours = oracle.exp_array(x)
    ref = np.exp(x.astype(np.float64)).astype(np.float32)
    normal = ref >= np.finfo(np.float32).tiny
    assert _ulp_diff(ours[normal], ref[normal]).max() <= 2
    assert oracle.exp_(0.0) == 1.0


def test_sigmoid_special_values_and_monotone():
    assert oracle.sigmoid(0.0) == 0.5
    assert oracle.sigmoid(100.0) == 1.0
    tiny = oracle.sigmoid(-100.0)
    assert 0.0 < tiny < 1e-37
    assert tiny == oracle.sigmoid(-88.0)                 # the argument clamp
    x = np.linspace(-40, 40, 1_000_001, dtype=np.float32)
    s = oracle.sigmoid_array(x)
    assert np.all(np.diff(s.astype(np.float64)) >= 0)
    ref = 1.0 / (1.0 + np.exp(-x.astype(np.float64)))
    assert np.max(np.abs(s - ref) / ref) < 4e-7


# ---------------------------------------------------------------- sum of squares
def test_sumsq_reduction_order_golden():
    for case, blocks, expected in _read_pairs("sumsq_order.txt"):
        parts = blocks.split("|")
        v = np.zeros(16 * len(parts), np.float32)
        for b, p in enumerate(parts):
            lead = [float(t) for t in p.split(",")]
            v[16 * b:16 * b + len(lead)] = lead
        assert float(oracle.sumsq(v)) == float(expected), case


def test_sumsq_constant_rows_closed_form():
    for a in (0.5, 1.0, 2.0, 0.25):
        for H in (16, 64, 1024, 8192, 16 * 3, 16 * 5):
            v = np.full(H, a, np.float32)
            assert float(oracle.sumsq(v)) == H * a * a


def test_sumsq_within_error_bound_of_exact_sum():
    rng = np.random.default_rng(11)
    for H in (16, 48, 1024, 2688, 8192):
        v = rng.standard_normal(H).astype(np.float32)
        exact = np.sum(v.astype(np.float64) ** 2)
        depth = 16 + int(np.ceil(np.log2(H // 16))) + 1
        assert abs(float(oracle.sumsq(v)) - exact) <= depth * 2.0 ** -24 * exact


def test_inv_rms_matches_float64_within_one_ulp():
    rng = np.random.default_rng(5)
    for _ in range(200):
        ss = np.float32(rng.random() * 1e4)
        H = int(rng.choice([16, 1024, 4096, 8192]))
        eps = np.float32(1e-6)
        ref = np.float32(1.0 / np.sqrt(np.float64(ss) / H + np.float64(eps)))
        got = oracle.inv_rms(ss, H, eps)
        assert _ulp_diff(np.array([got]), np.array([ref])).max() <= 2
