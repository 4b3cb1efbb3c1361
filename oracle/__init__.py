"""CPU oracle of the per-token MoE boundary (route, RMSNorm + NVFP4, combine, join).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  The product path
(``expert_combine_b200`` and its CUDA library) never imports, links or calls it.

The arithmetic lives in ``oracle.c`` (plain C, one IEEE binary32 operation per
source operation, no contraction); this module compiles it with gcc on first
use and marshals numpy arrays through ctypes.  Each wrapper names the passage
it follows; the C file repeats the citations next to the code.

Parity pins: every function here is pinned by ``tests/test_oracle_*.py`` against
format definitions, closed forms, library routines and brute force.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

CFLAGS = ["-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
          "-fno-fast-math", "-D_GNU_SOURCE"]


def build(force: bool = False) -> str:
    """Compile ``oracle.c`` into ``liboracle.so`` beside it (gcc, OpenMP)."""
    stale = (not os.path.exists(_LIB_PATH)
             or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC))
    if force or stale:
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.run(["gcc", *CFLAGS, _SRC, "-o", tmp, "-lm"], check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            # MB_ORACLE_LIB names another compiled copy of oracle.c to load
            # instead (the mutation tests point it at deliberately broken ones)
            lib = ctypes.CDLL(os.environ.get("MB_ORACLE_LIB") or build())
            P = ctypes.c_void_p
            i32, i64, f32 = ctypes.c_int, ctypes.c_int64, ctypes.c_float
            sig = {
                "oc_set_threads": (None, [i32]),
                "oc_get_threads": (i32, []),
                "oc_bf16_rn": (ctypes.c_uint16, [f32]),
                "oc_bf16_to_f32": (f32, [ctypes.c_uint16]),
                "oc_e4m3_rn_sat": (ctypes.c_uint8, [f32]),
                "oc_e4m3_decode": (f32, [ctypes.c_uint8]),
                "oc_e2m1_code": (ctypes.c_uint8, [f32]),
                "oc_exp": (f32, [f32]),
                "oc_sigmoid": (f32, [f32]),
                "oc_sumsq": (f32, [P, i32]),
                "oc_inv_rms": (f32, [f32, i32, f32]),
                "oc_route": (None, [P, P, P, i32, i32, i32, P, P]),
                "oc_norm_bf16": (None, [P, i32, i32, i32, P, f32, f32, P]),
                "oc_norm_quant": (None, [P, i32, i32, i32, P, f32, f32, f32, P, P, P]),
                "oc_combine": (None, [P, i64, i32, P, P, i32, i32, P, f32, f32, P]),
                "oc_join": (None, [P, P, P, f32, f32, f32, P, f32, f32, P, i32, i32, P]),
                "oc_dispatch": (None, [P, i32, i32, i32, i32, P, P, P]),
                "oc_router_logits": (None, [P, i32, i32, P, i32, f32, P, P]),
                "oc_finalize_allreduce": (None, [P, P, i32, i32, P, P, i32, i32, P, f32, f32, P, P]),
                "oc_bf16_rn_n": (None, [P, i64, P]),
                "oc_e4m3_rn_sat_n": (None, [P, i64, P]),
                "oc_e2m1_code_n": (None, [P, i64, P]),
                "oc_exp_n": (None, [P, i64, P]),
                "oc_sigmoid_n": (None, [P, i64, P]),
            }
            for name, (res, args) in sig.items():
                fn = getattr(lib, name)
                fn.restype = res
                fn.argtypes = args
            _lib = lib
    return _lib


def _ptr(a: np.ndarray | None):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


# ---------------------------------------------------------------- scalars
def set_threads(n: int) -> None:
    _load().oc_set_threads(int(n))


def get_threads() -> int:
    return int(_load().oc_get_threads())


def bf16_rn(x: float) -> int:
    return int(_load().oc_bf16_rn(float(x)))


def bf16_to_f32(b: int) -> float:
    return float(_load().oc_bf16_to_f32(int(b)))


def e4m3_rn_sat(x: float) -> int:
    """E4M3 round-to-nearest-even, saturating (prepare_trtllm_nvfp4, scale cast)."""
    return int(_load().oc_e4m3_rn_sat(float(x)))


def e4m3_decode(c: int) -> float:
    return float(_load().oc_e4m3_decode(int(c)))


def e2m1_code(q: float) -> int:
    """E2M1 threshold code (prepare_trtllm_nvfp4, _quantize_nvfp4_global_scale)."""
    return int(_load().oc_e2m1_code(float(q)))


def exp_(x: float) -> float:
    return float(_load().oc_exp(float(x)))


def sigmoid(x: float) -> float:
    return float(_load().oc_sigmoid(float(x)))


def _elementwise(name, x, out_dtype):
    x = _c(x, np.float32)
    out = np.empty(x.shape, out_dtype)
    getattr(_load(), name)(_ptr(x), int(x.size), _ptr(out))
    return out


def bf16_rn_array(x):
    """Element-wise BF16 round-to-nearest-even -> uint16 bits."""
    return _elementwise("oc_bf16_rn_n", x, np.uint16)


def e4m3_rn_sat_array(x):
    return _elementwise("oc_e4m3_rn_sat_n", x, np.uint8)


def e2m1_code_array(q):
    return _elementwise("oc_e2m1_code_n", q, np.uint8)


def exp_array(x):
    return _elementwise("oc_exp_n", x, np.float32)


def sigmoid_array(x):
    return _elementwise("oc_sigmoid_n", x, np.float32)


def sumsq(v) -> np.float32:
    v = _c(v, np.float32)
    assert v.size % 16 == 0
    return np.float32(_load().oc_sumsq(_ptr(v), int(v.size)))


def inv_rms(ss: float, H: int, eps: float) -> np.float32:
    return np.float32(_load().oc_inv_rms(float(ss), int(H), float(eps)))


# ---------------------------------------------------------------- stages
def route(logits, bias, mask, k: int):
    """Router gate (Muse Spark Open fast paths, Routing; MoE gate v2, token mask).

    logits float32 [T, E], bias float32 [E], mask uint8 [T] -> (ids int32 [T, k],
    weights float32 [T, k]).
    """
    logits = _c(logits, np.float32)
    T, E = logits.shape
    bias = _c(bias, np.float32)
    mask = _c(mask, np.uint8)
    assert bias.shape == (E,) and mask.shape == (T,) and 1 <= k <= E
    ids = np.empty((T, k), np.int32)
    w = np.empty((T, k), np.float32)
    _load().oc_route(_ptr(logits), _ptr(bias), _ptr(mask), T, E, k, _ptr(ids), _ptr(w))
    return ids, w


def norm_bf16(x, M: int, H: int, tp: int, w, gc: float, eps: float):
    """Weight-first RMSNorm rounded once to BF16 -> uint16 [M, H]."""
    x = _c(x, np.uint16).reshape(-1)
    w = _c(w, np.uint16)
    assert x.size == M * H and w.shape == (H,) and H % tp == 0 and (H // tp) % 16 == 0
    y = np.empty((M, H), np.uint16)
    _load().oc_norm_bf16(_ptr(x), M, H, tp, _ptr(w), float(gc), float(eps), _ptr(y))
    return y


def norm_quant(x, M: int, H: int, tp: int, w, gc: float, eps: float, gs: float,
               return_near: bool = False):
    """RMSNorm + NVFP4 (prepare_trtllm_nvfp4, norm_quant_trtllm_nvfp4).

    x uint16 (BF16 bits): [M, H] when tp == 1, else rank-block [tp, M, H/tp].
    Returns packed uint8 [M, H/2], sf uint8 [M, H/16] (and the near-threshold
    counts (codes, scales) when ``return_near``).
    """
    x = _c(x, np.uint16).reshape(-1)
    w = _c(w, np.uint16)
    assert x.size == M * H and w.shape == (H,) and H % tp == 0 and (H // tp) % 16 == 0
    packed = np.empty((M, H // 2), np.uint8)
    sf = np.empty((M, H // 16), np.uint8)
    near = np.zeros(2, np.int64)
    _load().oc_norm_quant(_ptr(x), M, H, tp, _ptr(w), float(gc), float(eps), float(gs),
                          _ptr(packed), _ptr(sf), _ptr(near))
    if return_near:
        return packed, sf, (int(near[0]), int(near[1]))
    return packed, sf


def combine(expert_out, R: int, row_idx, wt, w, gc: float, eps: float):
    """Post-expert norm + weighted combine (Muse Spark Open fast paths).

    expert_out uint16 [>=R, H] (rows at index >= R are never read), row_idx
    int32 [T, k], wt float32 [T, k], w uint16 [H] -> out uint16 [T, H].
    """
    expert_out = _c(expert_out, np.uint16)
    H = expert_out.shape[1]
    row_idx = _c(row_idx, np.int32)
    wt = _c(wt, np.float32)
    T, k = row_idx.shape
    assert wt.shape == (T, k) and expert_out.shape[0] >= R
    w = _c(w, np.uint16)
    out = np.empty((T, H), np.uint16)
    _load().oc_combine(_ptr(expert_out), int(R), H, _ptr(row_idx), _ptr(wt), T, k, _ptr(w),
                       float(gc), float(eps), _ptr(out))
    return out


def finalize_allreduce(expert_outs, Rs, row_idx, wt, w, gc: float, eps: float):
    """Expert finalize + tensor-parallel all-reduce (TensorRT-LLM PR 21356,
    "Fused finalize + all-reduce"; PR 21042, MoE paragraph).

    expert_outs: one uint16 [>=R_r, H] array per rank (rows at index >= R_r are
    never read); Rs: the ranks' row counts; row_idx int32 [world, T, k] (the
    local row of each slot, -1 where the expert is elsewhere); wt float32 [T, k];
    w uint16 [H].  Returns (out uint16 [T, H], partials float32 [world, T, H]).
    """
    world = len(expert_outs)
    assert len(Rs) == world
    eos = [_c(e, np.uint16) for e in expert_outs]
    H = eos[0].shape[1]
    assert all(e.shape[1] == H and e.shape[0] >= R for e, R in zip(eos, Rs))
    row_idx = _c(row_idx, np.int32)
    assert row_idx.shape[0] == world
    T, k = row_idx.shape[1], row_idx.shape[2]
    wt = _c(wt, np.float32)
    assert wt.shape == (T, k)
    w = _c(w, np.uint16)
    ptrs = (ctypes.c_void_p * world)(*[e.ctypes.data for e in eos])
    rs = np.asarray(Rs, np.int64)
    out = np.empty((T, H), np.uint16)
    partials = np.empty((world, T, H), np.float32)
    _load().oc_finalize_allreduce(ctypes.cast(ptrs, ctypes.c_void_p), _ptr(rs), world, H, _ptr(row_idx),
                                  _ptr(wt), T, k, _ptr(w), float(gc), float(eps), _ptr(partials),
                                  _ptr(out))
    return out, partials


def join(residual, branch, gain, alpha: float, beta: float, eps: float,
         next_w=None, next_gc: float = 1.0, next_eps: float = 1e-6, return_normed: bool = False):
    """Gated residual join (+ next prenorm), Muse Spark Open fast paths.

    Returns (new residual float32 [T, H], next prenorm uint16 [T, H] or None),
    and with ``return_normed`` also the BF16 bits of the normed branch term n
    (uint16 [T, H]) that enters the residual as beta * n.
    """
    r = np.array(residual, dtype=np.float32, copy=True, order="C")
    T, H = r.shape
    branch = _c(branch, np.uint16)
    gain = _c(gain, np.uint16)
    assert branch.shape == (T, H) and gain.shape == (H,)
    p = None
    nw = None
    if next_w is not None:
        nw = _c(next_w, np.uint16)
        p = np.empty((T, H), np.uint16)
    n = np.empty((T, H), np.uint16) if return_normed else None
    _load().oc_join(_ptr(r), _ptr(branch), _ptr(gain), float(alpha), float(beta), float(eps),
                    _ptr(nw), float(next_gc), float(next_eps), _ptr(p), T, H, _ptr(n))
    if return_normed:
        return r, p, n
    return r, p


def dispatch(ids, e0: int, E: int):
    """Expert-grouped rows of the routing entries (lmdeploy PR 4835 "MoE gate
    v2", commit notes: per-expert histogram and scan; en2f = -1 where no row).

    ``ids`` int32 [T, k] of global expert ids; experts [e0, e0 + E) are this
    rank's.  Returns ``offsets`` [E + 1], ``row_idx`` [T, k] (en2f) and
    ``row_token`` [T * k] (token of each row, -1 past the last row)."""
    ids = _c(ids, np.int32)
    T, k = ids.shape
    offsets = np.empty(E + 1, dtype=np.int32)
    row_idx = np.empty((T, k), dtype=np.int32)
    row_token = np.empty(T * k, dtype=np.int32)
    _load().oc_dispatch(_ptr(ids), T, k, e0, E, _ptr(offsets), _ptr(row_idx), _ptr(row_token))
    return offsets, row_idx, row_token


def router_logits(x_bf16, W, scale: float = 1.0):
    """Router projection in binary64 (TensorRT-LLM PR 21356, description,
    "Router projection": FP32 weights, FP32 accumulation, BF16 input cast,
    scale folded in).

    ``x_bf16`` uint16 [T, H] (BF16 bits), ``W`` float32 [E, H].  Returns
    (logits float64 [T, E], abs_sum float64 [T, E]) with abs_sum the sum of
    |scale * x * W| (the size of the rounding error of an FP32 evaluation)."""
    x = _c(x_bf16, np.uint16)
    W = _c(W, np.float32)
    T, H = x.shape
    E = W.shape[0]
    out = np.empty((T, E), dtype=np.float64)
    ab = np.empty((T, E), dtype=np.float64)
    _load().oc_router_logits(_ptr(x), T, H, _ptr(W), E, float(scale), _ptr(out), _ptr(ab))
    return out, ab
