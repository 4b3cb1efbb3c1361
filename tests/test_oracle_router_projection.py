"""Pins of the oracle's router projection (TensorRT-LLM PR 21356, description,
"Router projection": FP32 weights and accumulation, BF16 input cast, scale
folded in), evaluated in binary64."""
import os
from fractions import Fraction

import numpy as np

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _bf16_bits(a):
    """float32 values that are exact BF16 -> their BF16 bits."""
    u = np.asarray(a, np.float32).view(np.uint32)
    assert np.all((u & 0xFFFF) == 0)
    return (u >> 16).astype(np.uint16)


def test_router_projection_worked_example():
    kv = {}
    with open(os.path.join(GOLDEN, "router_projection_worked.txt")) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                key, *vals = line.split()
                kv[key] = vals
    x = np.array([int(v, 16) for v in kv["x_bits"]], np.uint16).reshape(2, 3)
    W = np.array(kv["W"], np.float32).reshape(2, 3)
    out, ab = oracle.router_logits(x, W, float(kv["scale"][0]))
    assert out.reshape(-1).tolist() == [float(v) for v in kv["logits"]]
    assert np.all(ab >= np.abs(out))


def test_router_projection_matches_float64_matmul():
    rng = np.random.default_rng(5)
    T, H, E = 37, 520, 19
    xf = rng.standard_normal((T, H)).astype(np.float32)
    x = (xf.view(np.uint32) >> 16).astype(np.uint16)         # truncate to BF16
    xb = (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    W = rng.standard_normal((E, H)).astype(np.float32)
    out, ab = oracle.router_logits(x, W, 0.75)
    want = 0.75 * (xb @ W.astype(np.float64).T)
    mag = 0.75 * (np.abs(xb) @ np.abs(W.astype(np.float64)).T)
    # two binary64 evaluations in different orders: within H ulps of the magnitude
    assert np.all(np.abs(out - want) <= H * 2.0 ** -52 * mag)
    assert np.allclose(ab, mag, rtol=1e-13)


def test_router_projection_exact_on_small_integers():
    # integers below 2^8 are exact in BF16 and FP32; sums below 2^53 are exact
    # in binary64, so the oracle must equal exact integer arithmetic
    rng = np.random.default_rng(9)
    T, H, E = 5, 300, 7
    xi = rng.integers(-100, 101, size=(T, H))
    Wi = rng.integers(-1000, 1001, size=(E, H))
    out, _ = oracle.router_logits(_bf16_bits(xi.astype(np.float32)), Wi.astype(np.float32), 1.0)
    want = [[sum(int(a) * int(b) for a, b in zip(xi[t], Wi[e])) for e in range(E)] for t in range(T)]
    assert out.tolist() == [[float(v) for v in row] for row in want]
    # the scale multiplies exactly when it is a power of two
    out2, _ = oracle.router_logits(_bf16_bits(xi.astype(np.float32)), Wi.astype(np.float32), 0.125)
    assert np.array_equal(out2, out * 0.125)


def test_router_projection_special_cases():
    x = np.zeros((3, 16), np.uint16)
    W = np.ones((4, 16), np.float32)
    out, ab = oracle.router_logits(x, W, 2.0)
    assert np.all(out == 0) and np.all(ab == 0)
    # one nonzero term: the product itself
    x[1, 5] = 0x4040                       # 3.0
    W[2, 5] = 1.5
    out, _ = oracle.router_logits(x, W, 1.0)
    assert out[1, 2] == 4.5 and out[1, 0] == 3.0 and out[0, 0] == 0.0
    # Fraction check of a non-integer case
    x2 = _bf16_bits(np.array([[0.375, -1.25]], np.float32))
    W2 = np.array([[0.1, 0.3]], np.float32)
    out, _ = oracle.router_logits(x2, W2, 1.0)
    exact = Fraction(0.375) * Fraction(float(W2[0, 0])) + Fraction(-1.25) * Fraction(float(W2[0, 1]))
    assert abs(Fraction(out[0, 0]) - exact) <= abs(exact) * Fraction(1, 2 ** 52)
