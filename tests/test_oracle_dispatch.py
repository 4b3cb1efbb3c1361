"""Pins of the oracle's dispatch (expert-grouped rows of the routing entries).

lmdeploy PR 4835 "MoE gate v2", commit notes: a per-expert histogram and scan
group the routing entries by expert; tokens without entries get no rows and
en2f is -1 there.  The oracle's counting sort is pinned against a hand-worked
example, numpy's stable argsort (a library routine) and invariants of the
layout.
"""
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden_cases():
    cases, k, ids, cur = [], None, None, None
    with open(os.path.join(GOLDEN, "dispatch_worked.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, *vals = line.split()
            if key == "k":
                k = int(vals[0])
            elif key == "ids":
                ids = np.array(vals, np.int32).reshape(-1, k)
            elif key == "case":
                cur = {"e0": int(vals[0]), "E": int(vals[1])}
                cases.append(cur)
            else:
                cur[key] = [int(v) for v in vals]
    return ids, cases


def test_dispatch_worked_example():
    ids, cases = _golden_cases()
    assert len(cases) == 2
    for c in cases:
        off, idx, tok = oracle.dispatch(ids, c["e0"], c["E"])
        assert off.tolist() == c["offsets"]
        assert idx.reshape(-1).tolist() == c["row_idx"]
        assert tok.tolist() == c["row_token"]


def _by_argsort(ids, e0, E):
    """The same layout from numpy's stable argsort of the local expert ids."""
    T, k = ids.shape
    flat = ids.reshape(-1).astype(np.int64) - e0
    valid = (flat >= 0) & (flat < E)
    pos = np.nonzero(valid)[0]
    order = pos[np.argsort(flat[pos], kind="stable")]
    R = order.size
    row_idx = np.full(T * k, -1, np.int64)
    row_idx[order] = np.arange(R)
    row_token = np.full(T * k, -1, np.int64)
    row_token[:R] = order // k
    offsets = np.concatenate([[0], np.cumsum(np.bincount(flat[pos], minlength=E))])
    return offsets, row_idx.reshape(T, k), row_token


@pytest.mark.parametrize("T,k,e0,E,seed", [
    (1, 1, 0, 1, 0), (7, 3, 0, 5, 1), (64, 8, 0, 256, 2), (300, 22, 0, 512, 3),
    (500, 8, 64, 64, 4), (129, 4, 3, 2, 5), (256, 8, 0, 2560, 6)])
def test_dispatch_matches_stable_argsort(T, k, e0, E, seed):
    rng = np.random.default_rng(seed)
    # global ids over a wider range than this rank's, with -1 entries and
    # repeated experts inside one token (the layout is defined for both)
    ids = rng.integers(-1, e0 + E + 3, size=(T, k)).astype(np.int32)
    ids[rng.random(T) < 0.1] = -1
    off, idx, tok = oracle.dispatch(ids, e0, E)
    r_off, r_idx, r_tok = _by_argsort(ids, e0, E)
    assert off.tolist() == r_off.tolist()
    assert np.array_equal(idx, r_idx)
    assert np.array_equal(tok, r_tok)


def test_dispatch_layout_invariants():
    rng = np.random.default_rng(11)
    T, k, E = 1000, 8, 256
    # router-like ids: k distinct experts per token, 5 % of tokens masked
    ids = np.stack([rng.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32)
    ids[rng.random(T) < 0.05] = -1
    off, idx, tok = oracle.dispatch(ids, 0, E)
    valid = ids >= 0
    R = int(valid.sum())
    assert off[0] == 0 and off[-1] == R and np.all(np.diff(off) >= 0)
    assert np.array_equal(np.diff(off), np.bincount(ids[valid], minlength=E))
    assert np.all(idx[~valid] == -1)
    # rows are a permutation of [0, R), and row_token inverts row_idx
    assert sorted(idx[valid].tolist()) == list(range(R))
    tt = np.nonzero(valid)[0]
    assert np.array_equal(tok[idx[valid]], tt)
    assert np.all(tok[R:] == -1)
    # each row lies in its expert's range; tokens ascend within an expert
    e_of_row = np.searchsorted(off, np.arange(R), side="right") - 1
    assert np.array_equal(e_of_row[idx[valid]], ids[valid])
    for e in range(E):
        seg = tok[off[e]:off[e + 1]]
        assert np.all(np.diff(seg) > 0)


def test_dispatch_special_cases():
    # nothing valid: empty ranges, every entry -1
    ids = np.full((5, 3), -1, np.int32)
    off, idx, tok = oracle.dispatch(ids, 0, 4)
    assert off.tolist() == [0] * 5 and np.all(idx == -1) and np.all(tok == -1)
    # k = 1 and expert = token: the identity layout
    T = 17
    ids = np.arange(T, dtype=np.int32).reshape(T, 1)
    off, idx, tok = oracle.dispatch(ids, 0, T)
    assert off.tolist() == list(range(T + 1))
    assert idx.reshape(-1).tolist() == list(range(T)) and tok.tolist() == list(range(T))
    # one expert takes every entry: rows follow the flattened order
    ids = np.zeros((4, 2), np.int32)
    ids[1, 1] = 5
    off, idx, tok = oracle.dispatch(ids, 0, 1)
    assert off.tolist() == [0, 7]
    assert idx.reshape(-1).tolist() == [0, 1, 2, -1, 3, 4, 5, 6]
    assert tok.tolist() == [0, 0, 1, 2, 2, 3, 3, -1]
