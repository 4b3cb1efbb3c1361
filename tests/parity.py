"""Shared helpers of the parity tests: run a stage on the GPU through the C ABI
and on the CPU oracle with the same inputs, and compare.

Expected values always come from ``oracle``; inputs come from
``expert_combine_b200.synth``.  Nothing here feeds a CUDA result to the oracle.
"""
from __future__ import annotations

import numpy as np
import torch

import expert_combine_b200 as eb
import oracle
from expert_combine_b200 import synth


def bf16_ulp_diff(a_u16, b_u16):
    """Distance in BF16 units in the last place between two bit arrays."""
    def key(u):
        u = np.asarray(u, np.uint16).astype(np.int32)
        return np.where(u & 0x8000, 0x8000 - (u & 0x7FFF), 0x8000 + u)
    return np.abs(key(a_u16) - key(b_u16))


def sample_tokens(T, n, seed=0, must=()):
    rng = np.random.default_rng(seed)
    pick = set(int(t) for t in must if 0 <= t < T)
    pick.update(rng.choice(T, size=min(n, T), replace=False).tolist())
    pick.update([0, T - 1])
    return np.array(sorted(pick), np.int64)


# ------------------------------------------------------------------ route
def check_route(case: synth.Case, tokens=None):
    ids, w = eb.moe_route(case.logits, case.bias, case.mask, case.k)
    torch.cuda.synchronize()
    if tokens is None:
        tokens = np.arange(case.T)
    tk = torch.as_tensor(tokens, device=case.logits.device)
    logits = synth.host(case.logits.index_select(0, tk))
    mask = synth.host(case.mask.index_select(0, tk))
    ids_o, w_o = oracle.route(logits, synth.host(case.bias), mask, case.k)
    ids_g = synth.host(ids.index_select(0, tk))
    w_g = synth.host(w.index_select(0, tk))
    assert np.array_equal(ids_g, ids_o), f"route ids differ at {np.argwhere(ids_g != ids_o)[:5]}"
    rel = np.abs(w_g.astype(np.float64) - w_o) / np.maximum(np.abs(w_o), 1e-30)
    assert np.all(rel <= 1e-6), f"route weights rel err {rel.max()}"
    return ids, w, int((w_g.view(np.uint32) != w_o.view(np.uint32)).sum())


# ------------------------------------------------------------------ norm-quant
def check_norm_quant(case: synth.Case, tokens=None):
    packed, sf = eb.norm_quant_nvfp4(case.x, case.T, case.norm_w, case.gc, case.eps, case.gs,
                                     tp=case.tp)
    torch.cuda.synchronize()
    gs = float(synth.host(case.gs)[0])
    if tokens is None:
        xh = synth.host(case.x)
        p_o, s_o, near = oracle.norm_quant(xh, case.T, case.H, case.tp, synth.host(case.norm_w),
                                           case.gc, case.eps, gs, return_near=True)
        p_g, s_g = synth.host(packed), synth.host(sf)
    else:
        tk = torch.as_tensor(tokens, device=case.x.device)
        xl = synth.host(case.x_logical().index_select(0, tk))
        p_o, s_o, near = oracle.norm_quant(xl, len(tokens), case.H, 1, synth.host(case.norm_w),
                                           case.gc, case.eps, gs, return_near=True)
        p_g = synth.host(packed.index_select(0, tk))
        s_g = synth.host(sf.index_select(0, tk))
    bad_p = int((p_g != p_o).sum())
    bad_s = int((s_g != s_o).sum())
    assert bad_p == 0 and bad_s == 0, (
        f"norm-quant mismatches: {bad_p} packed bytes, {bad_s} scales "
        f"(near-threshold codes {near[0]}, scales {near[1]})")
    return packed, sf, near


# ------------------------------------------------------------------ combine
def _gather_rows(case: synth.Case, tokens):
    """Rows the sampled tokens read, re-indexed densely (slot validity kept)."""
    idx = synth.host(case.row_idx)[tokens]
    valid = (idx >= 0) & (idx < case.R)
    rows = np.unique(idx[valid])
    rows_t = torch.as_tensor(rows, device=case.expert_buf.device, dtype=torch.int64)
    sub = synth.host(case.expert_out.index_select(0, rows_t)) if rows.size else \
        np.zeros((0, case.H), np.uint16)
    remap = np.full(idx.shape, -1, np.int32)
    remap[valid] = np.searchsorted(rows, idx[valid]).astype(np.int32)
    return sub, remap


def oracle_combine(case: synth.Case, wt_host, tokens=None):
    if tokens is None:
        G, R = case.guard, case.R
        buf = synth.host(case.expert_buf)
        return oracle.combine(buf[G:], R, synth.host(case.row_idx), wt_host,
                              synth.host(case.post_w), case.post_gc, case.eps)
    sub, remap = _gather_rows(case, tokens)
    return oracle.combine(sub, sub.shape[0], remap, wt_host[tokens], synth.host(case.post_w),
                          case.post_gc, case.eps)


def check_combine_rows(got_u16, rows_u16, R, row_idx, wt, post_w_u16, gc, eps):
    """A combine output against the oracle's combine of the same rows."""
    want = oracle.combine(rows_u16, R, row_idx, wt, post_w_u16, gc, eps)
    d = bf16_ulp_diff(got_u16, want)
    assert d.max() <= 1, f"combine differs by {d.max()} BF16 ulp at {np.argwhere(d > 1)[:5]}"
    return int((d > 0).sum())


def check_combine(case: synth.Case, tokens=None, wt=None, wt_host=None):
    if wt is None:
        wt = case.comb_wt
        wt_host = synth.host(case.comb_wt)
    out = eb.expert_combine(case.expert_out, case.R, case.row_idx, wt, case.post_w, case.post_gc,
                            case.eps)
    torch.cuda.synchronize()
    want = oracle_combine(case, wt_host, tokens)
    got = synth.host(out) if tokens is None else synth.host(
        out.index_select(0, torch.as_tensor(tokens, device=out.device)))
    d = bf16_ulp_diff(got, want)
    assert d.max() <= 1, f"combine differs by {d.max()} BF16 ulp at {np.argwhere(d > 1)[:5]}"
    return out, int((d > 0).sum())


# ------------------------------------------------------------------ join
def bf16_step(u16):
    """One BF16 unit in the last place at each value (bit patterns in, float64 out)."""
    e = (np.asarray(u16, np.uint16).astype(np.int64) >> 7) & 0xFF
    return np.where(e == 0, 2.0 ** -133, np.ldexp(1.0, (np.maximum(e, 1) - 127 - 7).astype(np.int32)))


def check_join_outputs(r_g, p_g, r_o, p_o, n_o, beta):
    """The join's outputs against the oracle's: the next prenorm within one
    BF16 step; the FP32 residual within 1e-5 relative, or within beta times
    one BF16 step of the normed term n at that element (n_o: the oracle's n,
    BF16 bits), the BF16 term that enters the FP32 stream (TensorRT-LLM
    PR 21356, description, gated residual join)."""
    if p_o is not None:
        d = bf16_ulp_diff(p_g, p_o)
        assert d.max() <= 1, f"prenorm differs by {d.max()} ulp"
    diff = np.abs(r_g.astype(np.float64) - r_o.astype(np.float64))
    rel = diff / np.maximum(np.abs(r_o.astype(np.float64)), 1e-30)
    ok = (rel <= 1e-5) | (diff <= abs(beta) * bf16_step(n_o))
    assert ok.all(), f"residual differs at {np.argwhere(~ok)[:5]}: rel err {rel[~ok].max()}"
    return int((r_g.view(np.uint32) != r_o.view(np.uint32)).sum())
