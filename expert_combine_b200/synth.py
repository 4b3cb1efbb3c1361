"""Seeded synthetic inputs for the MoE boundary, shaped like the pages' workloads.

This module holds input generation only -- none of the boundary's arithmetic.
Tests feed the same tensors to the CUDA path and (copied to the host) to the
CPU oracle; the benchmark uses it for its resident inputs.

Workloads (tokens T, hidden H, experts E, top-k):

===========  ======  =====  =====  ==  ====================================
name          T       H      E     k   notes
===========  ======  =====  =====  ==  ====================================
tiny          16      1024   256   8   3 exact score ties, 2 masked tokens,
                                       2 slots -1, 1 slot past the end
decode        128     8192   256   8   contiguous input, gated residual
                                       join + next prenorm fused
prefill       8192    8192   256   8   logits N(0,2), 1% slots -1, 5% of
                                       tokens masked
large_e       32768   4096   2560  8   bias U(-0.05,0.05), input in the
                                       rank-block layout [4, M, H/4]
wide_topk     65536   1024   512   22  bias 0, expert rows N(0, 0.5)
===========  ======  =====  =====  ==  ====================================

Every invalid slot and past-the-end slot points at NaN-filled guard rows, and
every masked token carries NaN logits, so a read of either poisons the output.
"""
from __future__ import annotations

import dataclasses
from typing import List, Optional

import torch

WORKLOADS = {
    "tiny": dict(T=16, H=1024, E=256, k=8, tp=1, logit_std=1.0, bias_range=0.1,
                 expert_std=1.0, mask_frac=0.0, slot_invalid_frac=0.0, join=True),
    "decode": dict(T=128, H=8192, E=256, k=8, tp=1, logit_std=1.0, bias_range=0.1,
                   expert_std=1.0, mask_frac=0.0, slot_invalid_frac=0.0, join=True),
    "prefill": dict(T=8192, H=8192, E=256, k=8, tp=1, logit_std=2.0, bias_range=0.1,
                    expert_std=1.0, mask_frac=0.05, slot_invalid_frac=0.01, join=False),
    "large_e": dict(T=32768, H=4096, E=2560, k=8, tp=4, logit_std=1.0, bias_range=0.05,
                    expert_std=1.0, mask_frac=0.0, slot_invalid_frac=0.0, join=False),
    "wide_topk": dict(T=65536, H=1024, E=512, k=22, tp=1, logit_std=1.0, bias_range=0.0,
                      expert_std=0.5, mask_frac=0.0, slot_invalid_frac=0.0, join=False),
}
SEEDS = {"tiny": 1001, "decode": 1002, "prefill": 1003, "large_e": 1004, "wide_topk": 1005}

# E4M3 max (448) times E2M1 max (6): the global scale maps the tensor's
# largest magnitude onto the top of both grids.
FP4_GLOBAL_NUMERATOR = 448.0 * 6.0

# Expert pairs whose bias values are made equal so that equal logits give
# exactly equal selection scores.
TIE_PAIRS = ((10, 11), (20, 21), (30, 31))


@dataclasses.dataclass
class Case:
    name: str
    T: int
    H: int
    E: int
    k: int
    tp: int
    # stage 1
    logits: torch.Tensor          # float32 [T, E]
    bias: torch.Tensor            # float32 [E]
    mask: torch.Tensor            # uint8 [T], 1 = valid token
    # stage 2
    x: torch.Tensor               # bfloat16, [T, H] or rank-block [tp, T, H/tp]
    norm_w: torch.Tensor          # bfloat16 [H]
    gc: float
    eps: float
    gs: torch.Tensor              # float32 [1]
    # stage 3
    expert_buf: torch.Tensor      # bfloat16 [G + R + G, H]; rows outside [G, G+R) are NaN
    guard: int                    # G
    R: int
    row_idx: torch.Tensor         # int32 [T, k]; -1 or >= R marks an invalid slot
    comb_wt: torch.Tensor         # float32 [T, k] (standalone combine weights)
    post_w: torch.Tensor          # bfloat16 [H]
    post_gc: float
    # gated residual join (None when the workload has no join)
    residual: Optional[torch.Tensor] = None   # float32 [T, H]
    gain: Optional[torch.Tensor] = None       # bfloat16 [H]
    next_w: Optional[torch.Tensor] = None     # bfloat16 [H]
    next_gc: float = 1.0
    alpha: float = 1.0
    beta: float = 0.5

    @property
    def expert_out(self) -> torch.Tensor:
        """The [R, H] view the combine receives (guard rows lie around it)."""
        return self.expert_buf[self.guard:self.guard + self.R]

    def x_logical(self) -> torch.Tensor:
        """The input as a logical [T, H] tensor (a copy for rank-block storage)."""
        if self.tp == 1:
            return self.x
        return self.x.permute(1, 0, 2).reshape(self.T, self.H)


def _normal(shape, std, gen, device, dtype=torch.float32, mean=0.0, chunk=1 << 26):
    out = torch.empty(shape, dtype=dtype, device=device)
    flat = out.view(-1)
    for s in range(0, flat.numel(), chunk):
        e = min(flat.numel(), s + chunk)
        tmp = torch.empty(e - s, dtype=torch.float32, device=device)
        tmp.normal_(mean, std, generator=gen)
        flat[s:e].copy_(tmp)
    return out


def _uniform(shape, lo, hi, gen, device):
    out = torch.empty(shape, dtype=torch.float32, device=device)
    out.uniform_(lo, hi, generator=gen)
    return out


def make_case(name: str, device="cpu", seed: Optional[int] = None, T: Optional[int] = None,
              H: Optional[int] = None, E: Optional[int] = None, k: Optional[int] = None,
              tp: Optional[int] = None, join: Optional[bool] = None, guard: int = 8,
              gc: float = 0.0) -> Case:
    """Build the named workload (sizes may be overridden for small variants).

    ``gc`` is the gain centre of the pre-expert norm: 0 means the BF16 weight is
    the gain itself (weights drawn N(1, 0.1)); 1 means the Gemma-style gain
    1 + w (weights then drawn N(0, 0.1)).
    """
    cfg = dict(WORKLOADS[name])
    for key, val in (("T", T), ("H", H), ("E", E), ("k", k), ("tp", tp), ("join", join)):
        if val is not None:
            cfg[key] = val
    T_, H_, E_, k_, tp_ = cfg["T"], cfg["H"], cfg["E"], cfg["k"], cfg["tp"]
    assert H_ % tp_ == 0 and (H_ // tp_) % 16 == 0 and k_ <= E_
    device = torch.device(device)
    gen = torch.Generator(device=device)
    gen.manual_seed(SEEDS[name] if seed is None else seed)

    # ---- stage 1 inputs
    logits = _normal((T_, E_), cfg["logit_std"], gen, device)
    if cfg["bias_range"] > 0:
        bias = _uniform((E_,), -cfg["bias_range"], cfg["bias_range"], gen, device)
    else:
        bias = torch.zeros(E_, dtype=torch.float32, device=device)
    mask = torch.ones(T_, dtype=torch.uint8, device=device)
    if name == "tiny" and T_ >= 12:
        mask[3] = 0
        mask[11] = 0
    elif name == "decode" and T_ >= 91:
        mask[17] = 0
        mask[90] = 0
    if cfg["mask_frac"] > 0:
        drop = _uniform((T_,), 0.0, 1.0, gen, device) < cfg["mask_frac"]
        mask[drop] = 0
    if name == "tiny" and E_ >= 32 and T_ >= 3 and k_ >= 3:
        for a, b in TIE_PAIRS:
            bias[b] = bias[a]
        # token 0: the tied pair straddles the k-th / (k+1)-th place;
        # token 1: both members inside the top-k; token 2: both far below.
        hi, mid, lo = 30.0, 0.0, -30.0
        logits[0].fill_(lo)
        top0 = [e for e in range(40, E_)][: k_ - 1]
        logits[0, top0] = hi
        logits[0, 10] = mid
        logits[0, 11] = mid
        logits[1].fill_(lo)
        top1 = [e for e in range(40, E_)][: k_ - 2]
        logits[1, top1] = hi
        logits[1, 20] = hi
        logits[1, 21] = hi
        logits[2, 30] = lo
        logits[2, 31] = lo
    logits[mask == 0] = float("nan")

    # ---- stage 2 inputs
    xl = _normal((T_, H_), 1.0, gen, device, dtype=torch.bfloat16)
    if tp_ == 1:
        x = xl
    else:
        x = xl.view(T_, tp_, H_ // tp_).permute(1, 0, 2).contiguous()
    w_mean = 1.0 if gc == 0.0 else 0.0
    norm_w = _normal((H_,), 0.1, gen, device, dtype=torch.bfloat16, mean=w_mean)
    amax = xl.abs().max().float() if xl.numel() else torch.tensor(1.0, device=device)
    gs = (torch.tensor(FP4_GLOBAL_NUMERATOR, dtype=torch.float32, device=device)
          / amax).reshape(1).to(torch.float32)
    del xl

    # ---- stage 3 inputs
    R = T_ * k_
    G = guard
    expert_buf = torch.full((G + R + G, H_), float("nan"), dtype=torch.bfloat16, device=device)
    if R:
        expert_buf[G:G + R] = _normal((R, H_), cfg["expert_std"], gen, device,
                                      dtype=torch.bfloat16)
    perm = torch.randperm(R, generator=gen, device=device).to(torch.int32)
    row_idx = perm.view(T_, k_).clone()
    if cfg["slot_invalid_frac"] > 0:
        bad = _uniform((T_, k_), 0.0, 1.0, gen, device) < cfg["slot_invalid_frac"]
        row_idx[bad] = -1
    if name == "tiny" and T_ >= 10 and k_ >= 6:
        row_idx[5, 2] = -1
        row_idx[7, 0] = -1
        row_idx[9, 5] = R + 3
    row_idx[mask == 0] = -1
    comb_wt = _uniform((T_, k_), 0.0, 0.25, gen, device)
    post_w = _normal((H_,), 0.1, gen, device, dtype=torch.bfloat16, mean=1.0)

    case = Case(name=name, T=T_, H=H_, E=E_, k=k_, tp=tp_, logits=logits, bias=bias,
                mask=mask, x=x, norm_w=norm_w, gc=gc, eps=1e-6, gs=gs,
                expert_buf=expert_buf, guard=G, R=R, row_idx=row_idx, comb_wt=comb_wt,
                post_w=post_w, post_gc=0.0)
    if cfg["join"]:
        case.residual = _normal((T_, H_), 1.0, gen, device)
        case.gain = _normal((H_,), 0.1, gen, device, dtype=torch.bfloat16, mean=1.0)
        case.next_w = _normal((H_,), 0.1, gen, device, dtype=torch.bfloat16)
        case.next_gc = 1.0
        case.alpha = 1.0
        case.beta = 0.5
    return case


def make_topk_ids(T: int, k: int, E: int, seed: int, masked_frac: float = 0.05,
                  invalid_frac: float = 0.0, expert_begin: int = 0, span: Optional[int] = None,
                  distinct: bool = True, device="cpu") -> torch.Tensor:
    """Router-shaped expert ids [T, k] int32 (dispatch input), seeded.

    Each token draws k experts from [expert_begin, expert_begin + span)
    (span defaults to E), distinct within the token unless ``distinct`` is
    False; ``masked_frac`` of the tokens are masked (all -1) and
    ``invalid_frac`` of the remaining slots are set to -1."""
    gen = torch.Generator(device="cpu")
    gen.manual_seed(seed)
    span = E if span is None else span
    ids = torch.empty(T, k, dtype=torch.int64)
    step = max(1, (1 << 24) // max(span, 1))
    for s in range(0, T, step):
        e = min(T, s + step)
        if distinct:
            keys = torch.rand(e - s, span, generator=gen)
            ids[s:e] = keys.topk(k, dim=1).indices
        else:
            ids[s:e] = torch.randint(0, span, (e - s, k), generator=gen)
    ids += expert_begin
    masked = torch.rand(T, generator=gen) < masked_frac
    ids[masked] = -1
    if invalid_frac > 0:
        ids[torch.rand(T, k, generator=gen) < invalid_frac] = -1
    return ids.to(torch.int32).to(device)


def as_u16(t: torch.Tensor):
    """BF16 tensor -> numpy uint16 array of its bits (host copy)."""
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view("uint16")


def host(t: torch.Tensor):
    """Any tensor -> numpy host copy (BF16 as uint16 bits)."""
    if t.dtype == torch.bfloat16:
        return as_u16(t)
    return t.detach().contiguous().cpu().numpy()


@dataclasses.dataclass
class EpCase:
    """Inputs of the expert finalize + all-reduce with the experts split over
    `world` ranks (expert e on rank e // (E / world)): per rank, the rows of
    its own slots (one BF16 N(0, 1) row per slot, in token-major slot order,
    followed by `nan_tail` NaN rows that must never be read) and its row
    indices (the local row, -1 for a slot of another rank's expert or of a
    masked token, and a few slots of other ranks pointing past the end)."""
    T: int
    H: int
    k: int
    E: int
    world: int
    ids: torch.Tensor                 # int32 [T, k] (-1: masked / absent)
    expert_out: List[torch.Tensor]    # per rank: bfloat16 [R_r + nan_tail, H]
    R: List[int]
    row_idx: List[torch.Tensor]       # per rank: int32 [T, k]
    weights: torch.Tensor             # float32 [T, k] (the same on every rank)
    norm_w: torch.Tensor              # bfloat16 [H]
    gc: float
    eps: float


def make_ep_case(T: int, H: int, k: int, E: int, world: int, seed: int, gc: float = 0.0,
                 masked_frac: float = 0.05, nan_tail: int = 2, device="cpu") -> EpCase:
    gen = torch.Generator(device="cpu")
    gen.manual_seed(seed)
    ids = make_topk_ids(T, k, E, seed, masked_frac=masked_frac, invalid_frac=0.01)
    per = (E + world - 1) // world
    owner = torch.where(ids >= 0, ids // per, torch.full_like(ids, -1))
    outs, Rs, idxs = [], [], []
    for r in range(world):
        mine = owner == r
        R = int(mine.sum())
        idx = torch.full((T, k), -1, dtype=torch.int32)
        idx[mine] = torch.arange(R, dtype=torch.int32)
        # some slots of other ranks point past this rank's rows (never read)
        elsewhere = (owner >= 0) & ~mine & (torch.rand(T, k, generator=gen) < 0.1)
        idx[elsewhere] = R + torch.randint(0, max(nan_tail, 1), (int(elsewhere.sum()),), generator=gen,
                                           dtype=torch.int32)
        rows = torch.empty(R + nan_tail, H, dtype=torch.bfloat16)
        rows[:R] = torch.randn(R, H, generator=gen).to(torch.bfloat16)
        rows[R:] = float("nan")
        outs.append(rows.to(device))
        Rs.append(R)
        idxs.append(idx.to(device))
    weights = torch.rand(T, k, generator=gen).to(device)
    mean = 1.0 if gc == 0.0 else 0.0
    norm_w = (mean + 0.1 * torch.randn(H, generator=gen)).to(torch.bfloat16).to(device)
    return EpCase(T, H, k, E, world, ids.to(device), outs, Rs, idxs, weights, norm_w, gc, 1e-6)
