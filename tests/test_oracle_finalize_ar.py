"""Pins of the oracle's expert finalize + tensor-parallel all-reduce
(TensorRT-LLM PR 21356, "Fused finalize + all-reduce"; PR 21042, MoE
paragraph): each rank's partial is the combine's FP32 accumulator over its own
experts' slots, the partials are added in FP32 in rank order, one BF16
rounding at the end.

The pins reach outside the function: with one rank it must equal the pinned
combine bit for bit; on inputs whose every sum is exact it must equal integer
arithmetic under any assignment of experts to ranks; and a case on a BF16
rounding tie shows the rank order of the FP32 sum."""
from fractions import Fraction

import numpy as np
import pytest

import oracle

BF16_ONE = 0x3F80


def bf16_bits(v: float) -> int:
    return oracle.bf16_rn(float(v))


def split_by_rank(rows_of_slot, owner, world, H, nan_tail=2):
    """Per-rank expert outputs and row indices for slots (t, j) whose row is
    rows_of_slot[t][j] (uint16 [H], or None for an absent slot) and whose
    expert lives on rank owner[t][j].  Each rank's array gets NaN rows past
    its row count (never to be read)."""
    T, k = len(rows_of_slot), len(rows_of_slot[0])
    outs, Rs = [], []
    idx = np.full((world, T, k), -1, np.int32)
    nan = np.full(H, 0x7FC0, np.uint16)
    for r in range(world):
        rows = []
        for t in range(T):
            for j in range(k):
                if rows_of_slot[t][j] is not None and owner[t][j] == r:
                    idx[r, t, j] = len(rows)
                    rows.append(rows_of_slot[t][j])
        R = len(rows)
        rows += [nan] * nan_tail
        outs.append(np.stack(rows) if rows else np.zeros((0, H), np.uint16))
        Rs.append(R)
    return outs, Rs, idx


def test_one_rank_is_the_combine():
    rng = np.random.default_rng(3)
    T, H, k, R = 9, 96, 5, 30
    eo = oracle.bf16_rn_array(rng.standard_normal((R + 3, H)).astype(np.float32))
    eo[R:] = 0x7FC0                                           # NaN rows past the end
    idx = rng.integers(-1, R + 3, (T, k)).astype(np.int32)   # -1 and >= R are invalid
    wt = rng.random((T, k)).astype(np.float32)
    w = oracle.bf16_rn_array((1 + 0.1 * rng.standard_normal(H)).astype(np.float32))
    for gc in (0.0, 1.0):
        want = oracle.combine(eo, R, idx, wt, w, gc, 1e-6)
        out, part = oracle.finalize_allreduce([eo], [R], idx[None], wt, w, gc, 1e-6)
        assert np.array_equal(out, want)
        assert np.array_equal(oracle.bf16_rn_array(part[0]), want)


def _exact_case(seed, T=12, k=8, H=64):
    """Rows of constant +-1 with a unit norm weight and a negligible eps make
    every normalised element exactly +-1; weights are multiples of 1/16, so
    every partial and every sum is exact and the result fits BF16."""
    rng = np.random.default_rng(seed)
    sign = rng.choice([-1.0, 1.0], (T, k))
    wq = rng.integers(1, 17, (T, k))
    present = rng.random((T, k)) > 0.15
    rows = [[oracle.bf16_rn_array(np.full(H, sign[t, j], np.float32)) if present[t, j] else None
             for j in range(k)] for t in range(T)]
    wt = (wq / 16.0).astype(np.float32)
    exact = [sum(Fraction(int(wq[t, j]), 16) * int(sign[t, j]) for j in range(k) if present[t, j])
             for t in range(T)]
    return rows, wt, exact, present


@pytest.mark.parametrize("world", [1, 2, 3, 4, 8])
@pytest.mark.parametrize("assign", ["blocks", "round_robin", "random"])
def test_any_expert_split_gives_the_exact_sum(world, assign):
    T, k, H = 12, 8, 64
    rows, wt, exact, _ = _exact_case(seed=world * 7 + len(assign), T=T, k=k, H=H)
    rng = np.random.default_rng(11)
    experts = rng.integers(0, 64, (T, k))
    if assign == "blocks":
        owner = experts // (64 // world + (64 % world > 0))
    elif assign == "round_robin":
        owner = experts % world
    else:
        owner = rng.integers(0, world, (T, k))
    outs, Rs, idx = split_by_rank(rows, owner, world, H)
    w = oracle.bf16_rn_array(np.ones(H, np.float32))
    out, part = oracle.finalize_allreduce(outs, Rs, idx, wt, w, 0.0, 2.0 ** -30)
    for t in range(T):
        want = bf16_bits(float(exact[t]))
        assert np.all(out[t] == want), (t, exact[t])
        # each partial is exactly the rank's own share
        for r in range(world):
            share = sum(float(wt[t, j]) * float(rows[t][j][0] == BF16_ONE and 1 or -1)
                        for j in range(k) if rows[t][j] is not None and owner[t, j] == r)
            assert np.all(part[r, t] == np.float32(share))


def test_partials_are_added_in_rank_order():
    """One token, three slots of rows that normalise to exactly 1, weights
    1 + 2^-8, 2^-24, 2^-24.  In rank order (big partial first) each small
    partial is a tie that rounds away and bf16(1 + 2^-8) is a tie to even:
    1.0.  With the big partial on the last rank the two small ones first make
    2^-23, the FP32 sum is 1 + 2^-8 + 2^-23, above the BF16 midpoint: 1 + 2^-7."""
    H = 32
    one = oracle.bf16_rn_array(np.ones(H, np.float32))
    rows = [[one, one, one]]
    wt = np.array([[1 + 2.0 ** -8, 2.0 ** -24, 2.0 ** -24]], np.float32)
    w = one
    for owner, want in (([[0, 1, 2]], BF16_ONE), ([[2, 0, 1]], BF16_ONE + 1)):
        outs, Rs, idx = split_by_rank(rows, np.array(owner), 3, H)
        out, part = oracle.finalize_allreduce(outs, Rs, idx, wt, w, 0.0, 2.0 ** -30)
        assert np.all(out == want), (owner, hex(int(out[0, 0])))
        for r in range(3):
            j = owner[0].index(r)
            assert np.all(part[r, 0] == wt[0, j])


def test_slots_elsewhere_or_past_the_end_are_never_read():
    """Slots pointing at -1 or past a rank's rows (NaN rows) contribute
    nothing; a token without a valid slot on any rank outputs +0."""
    T, k, H = 12, 8, 64
    rows, wt, exact, present = _exact_case(seed=5, T=T, k=k, H=H)
    rows[4] = [None] * k                       # token 4: no slot on any rank
    exact[4] = 0
    owner = np.tile(np.arange(k) % 2, (T, 1))
    outs, Rs, idx = split_by_rank(rows, owner, 2, H, nan_tail=3)
    # redirect absent slots to the NaN rows past the end instead of -1
    for r in range(2):
        absent = idx[r] < 0
        idx[r][absent & (np.arange(k)[None, :] % 2 == 0)] = Rs[r] + 1
    w = oracle.bf16_rn_array(np.ones(H, np.float32))
    out, part = oracle.finalize_allreduce(outs, Rs, idx, wt, w, 0.0, 2.0 ** -30)
    assert np.all(np.isfinite(part))
    for t in range(T):
        assert np.all(out[t] == bf16_bits(float(exact[t])))
    assert np.all(out[4] == 0)
