#!/usr/bin/env python
"""Throughput of the MoE boundary step: router gate + RMSNorm/NVFP4 + post-expert combine.

Workload (one step, per GPU): T=8192 tokens, H=8192, E=256 experts, top-8,
router logits FP32 N(0, 2), 5% of tokens masked, 1% of expert slots invalid,
expert outputs [T*8, H] BF16 -- synthetic, seeded, resident in HBM.  The
calls go through the library's C ABI on one stream: moe_route_norm_quant (the
router and the pre-expert norm-quant of the same tokens) and expert_combine;
`--separate` issues moe_route and norm_quant_nvfp4 as two calls instead.

  python bench.py [--gpus N --steps K --warmup W] [--impl reference]

Prints ONE JSON line (rank 0).  `value` is tokens/s over all ranks (weak
scaling: every rank runs its own batch of 8192 tokens).  The per-step inputs
(1.2 GB) are larger than the 126 MB L2, so no flush runs between steps.

Timing: the K steps are captured once in a CUDA graph (the library's calls
are capture-safe) and the timed region replays it between two CUDA events on
the launching stream (barrier + synchronize on both sides, max over ranks), so
the number is the GPU's and not the Python launch path's; no event sits between
the kernels of the region, since one would keep the next kernel from launching
early.  The same K steps launched one call at a time from Python are timed too
(`stream_launch`).  The per-stage times (`stages_ms`, and the combine's launch
duration in `roofline`) come from graphs of K launches of one stage.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from expert_combine_b200 import shard  # noqa: E402

WORKLOAD = "prefill"
METRIC = "tokens/s of route+norm-quant+combine at 8192 tok, H=8192; HBM GB/s vs 8 TB/s"
NOMINAL_HBM_GBS = 8000.0


def bytes_per_token(H, E, k):
    """Algorithmic bytes per token, counted once (reads + writes)."""
    route = 4 * E + 1 + 8 * k                       # logits, mask, ids + weights
    norm_quant = 2 * H + H // 2 + H // 16           # x, packed codes, scales
    combine = 2 * k * H + 8 * k + 2 * H             # k expert rows, idx + weights, out
    return route, norm_quant, combine


# DRAM traffic of one combine launch: dram__bytes_read.sum +
# dram__bytes_write.sum from one ncu capture of a single combine_wide launch on
# the prefill workload cut to 2048 tokens (profiles/combine_wide_prefill_T2048_
# H8192_traffic.md), scaled to a launch of this bench by the algorithmic bytes
# (the reads equal the algorithmic reads there, so the traffic grows with the
# rows read).  It stands only while the kernel's sources hash to `src`;
# otherwise it is reported null.
COMBINE_TRAFFIC = {"src": "adf132b0c0f7fea9", "tokens": 2048, "bytes": 251288832 + 20741888,
                   "algorithmic_bytes": 284786688}
COMBINE_SOURCES = ("combine.cu", "ring.cuh", "common.cuh", "tmem.cuh")


def combine_traffic(algorithmic_bytes):
    import hashlib
    h = hashlib.sha256()
    for name in COMBINE_SOURCES:
        with open(os.path.join(ROOT, "expert_combine_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    if h.hexdigest()[:16] != COMBINE_TRAFFIC["src"]:
        return None
    return int(round(COMBINE_TRAFFIC["bytes"] * algorithmic_bytes / COMBINE_TRAFFIC["algorithmic_bytes"]))


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap,clocks.mem,"
              "power.limit")

    def __init__(self, device_index):
        self.idx = device_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        self.out = ""
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        rows = []
        for line in (self.out or "").strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 9:
                rows.append(parts)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        smax = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i] == "Active"})
        num = lambda v: v.replace(".", "").isdigit()
        mem = [float(r[9]) for r in rows if len(r) > 9 and num(r[9])]
        pw = [float(r[3]) for r in rows if num(r[3])]
        lim = [float(r[10]) for r in rows if len(r) > 10 and num(r[10])]
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None, "reasons": reasons,
                "samples": len(rows), "mem_mhz": statistics.median(mem) if mem else None,
                "power_w_max": max(pw) if pw else None, "power_limit_w": min(lim) if lim else None}


# ---------------------------------------------------------------------------- CPU oracle
def oracle_step(case_host, tokens):
    """The oracle on a sample of the workload's tokens (all three stages)."""
    import oracle
    c = case_host
    ids, w = oracle.route(c["logits"][tokens], c["bias"], c["mask"][tokens], c["k"])
    oracle.norm_quant(c["x"][tokens], len(tokens), c["H"], 1, c["norm_w"], c["gc"], c["eps"],
                      c["gs"])
    idx = c["row_idx"][tokens]
    valid = (idx >= 0) & (idx < c["R"])
    rows = np.unique(idx[valid])
    remap = np.full(idx.shape, -1, np.int32)
    remap[valid] = np.searchsorted(rows, idx[valid]).astype(np.int32)
    sub = c["expert_rows"](rows)
    oracle.combine(sub, sub.shape[0], remap, w, c["post_w"], c["post_gc"], c["eps"])


def host_sample(case, n_tokens, seed=0):
    """Copy to the host what the oracle needs for a sample of tokens."""
    from expert_combine_b200 import synth
    rng = np.random.default_rng(seed)
    tokens = np.sort(rng.choice(case.T, size=n_tokens, replace=False))
    tk = torch.as_tensor(tokens, device=case.logits.device)
    idx = synth.host(case.row_idx)
    sel_rows = idx[tokens]
    need = np.unique(sel_rows[(sel_rows >= 0) & (sel_rows < case.R)])
    rows_host = synth.host(case.expert_out.index_select(
        0, torch.as_tensor(need, device=case.logits.device, dtype=torch.int64)))
    logits = np.full((case.T, case.E), np.nan, np.float32)
    logits[tokens] = synth.host(case.logits.index_select(0, tk))
    x = np.zeros((case.T, case.H), np.uint16)
    x[tokens] = synth.host(case.x_logical().index_select(0, tk))

    def expert_rows(rows):
        pos = np.searchsorted(need, rows)
        return rows_host[pos]

    return tokens, dict(logits=logits, bias=synth.host(case.bias), mask=synth.host(case.mask),
                        k=case.k, x=x, H=case.H, norm_w=synth.host(case.norm_w), gc=case.gc,
                        eps=case.eps, gs=float(synth.host(case.gs)[0]), row_idx=idx, R=case.R,
                        expert_rows=expert_rows, post_w=synth.host(case.post_w),
                        post_gc=case.post_gc)


def near_threshold_report(case, packed, sf):
    """NVFP4 values of the whole batch whose FP32 pre-quantisation value (or
    the scale's FP32 argument) lies within one ulp of a rounding threshold,
    counted by the oracle over every token, and how many of the GPU's codes and
    scales differ from the oracle's (part of the CPU-baseline leg: the only
    place the benchmark runs the oracle)."""
    import oracle
    from expert_combine_b200 import synth
    p_o, s_o, near_ = oracle.norm_quant(synth.host(case.x), case.T, case.H, case.tp, synth.host(case.norm_w),
                                        case.gc, case.eps, float(synth.host(case.gs)[0]), return_near=True)
    return {"codes_near": near_[0], "scales_near": near_[1], "codes": case.T * case.H,
            "scales": case.T * case.H // 16,
            "packed_bytes_differing": int((synth.host(packed) != p_o).sum()),
            "scales_differing": int((synth.host(sf) != s_o).sum()),
            "how": "oracle over all tokens of the step's batch; the GPU's outputs of the last timed step"}


def time_oracle(case_host, tokens, budget_s=15.0):
    import oracle
    cores = oracle.get_threads()
    t0 = time.perf_counter()
    oracle_step(case_host, tokens)
    one = time.perf_counter() - t0
    reps = max(1, min(20, int(budget_s / max(one, 1e-3))))
    times = [one]
    for _ in range(reps - 1):
        t0 = time.perf_counter()
        oracle_step(case_host, tokens)
        times.append(time.perf_counter() - t0)
    med = statistics.median(times)
    return len(tokens) / med, cores, reps, med


def prefill_config(case, world):
    """The `config` of the JSON line: the prefill workload, the same on both arms."""
    from expert_combine_b200 import synth
    idx_h = synth.host(case.row_idx)
    return {"workload": f"prefill T={case.T} H={case.H} E={case.E} k={case.k} (route+norm-quant+combine)",
            "tokens_per_rank": case.T, "hidden": case.H, "experts": case.E, "top_k": case.k,
            "expert_rows": case.R, "valid_tokens": int(synth.host(case.mask).sum()),
            "valid_slots": int(((idx_h >= 0) & (idx_h < case.R)).sum()), "parallelism": f"dp{world}",
            "l2": "inputs larger than L2 (1.2 GB per step), no flush"}


# ---------------------------------------------------------------------------- reference arm
def run_reference(args, info):
    if info.rank != 0:
        return 0
    from expert_combine_b200 import synth
    case = synth.make_case(WORKLOAD, device="cuda" if torch.cuda.is_available() else "cpu",
                           seed=shard.rank_seed(synth.SEEDS[WORKLOAD], info), T=args.tokens)
    n_sample = min(256, case.T)
    tokens, ch = host_sample(case, n_sample, seed=1)
    import oracle
    cores = oracle.get_threads()
    for _ in range(args.warmup):
        oracle_step(ch, tokens)
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        oracle_step(ch, tokens)
        times.append(time.perf_counter() - t0)
    per_step = sum(times) / len(times)
    value = len(tokens) / per_step
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": per_step * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": prefill_config(case, info.world),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": f"{n_sample} of {case.T} tokens per step (all three stages), "
                                   f"scaled to the metric's unit"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------- our arm
def run_ours(args, info):
    world, rank, local = info.world, info.rank, info.local
    import expert_combine_b200 as eb
    from expert_combine_b200 import synth

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    eb.load()
    case = synth.make_case(WORKLOAD, device=dev, seed=shard.rank_seed(synth.SEEDS[WORKLOAD], info),
                           T=args.tokens)
    T, H, E, k = case.T, case.H, case.E, case.k
    ids = torch.empty(T, k, dtype=torch.int32, device=dev)
    w = torch.empty(T, k, dtype=torch.float32, device=dev)
    packed = torch.empty(T, H // 2, dtype=torch.uint8, device=dev)
    sf = torch.empty(T, H // 16, dtype=torch.uint8, device=dev)
    out = torch.empty(T, H, dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream(dev)

    def pre_expert():
        # the router gate and the pre-expert RMSNorm + NVFP4 of the same tokens
        if args.separate:
            eb.moe_route(case.logits, case.bias, case.mask, k, ids, w)
            eb.norm_quant_nvfp4(case.x, T, case.norm_w, case.gc, case.eps, case.gs, packed=packed,
                                sf=sf)
        else:
            eb.moe_route_norm_quant(case.logits, case.bias, case.mask, k, case.x, case.norm_w,
                                    case.gc, case.eps, case.gs, topk_ids=ids, topk_weights=w,
                                    packed=packed, sf=sf)

    pre_kernels = 2 if args.separate else eb.route_norm_quant_kernels(T, H, E, k, tp=case.tp)

    def combine():
        eb.expert_combine(case.expert_out, case.R, case.row_idx, w, case.post_w, case.post_gc,
                          case.eps, out=out)

    def step():
        pre_expert()
        combine()

    def timed(fn, n):
        # n back-to-back calls between two events on the launching stream; an
        # event between kernels would stop the next kernel's early launch, so
        # none is recorded inside the region
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for _ in range(n):
            fn()
        t1.record(stream)
        return t0, t1

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if eb.device_status() != 0:
        raise RuntimeError("a kernel reported a wait timeout during warm-up")
    g_step = capture_graph(step, args.steps, dev)
    g_pre = capture_graph(pre_expert, args.steps, dev)
    g_cmb = capture_graph(combine, args.steps, dev)
    for g in (g_step, g_pre, g_cmb):                  # untimed: each graph's first launch uploads it
        g.replay()
    torch.cuda.synchronize()

    shard.barrier(info)
    torch.cuda.synchronize()
    with ClockSampler(dev.index) as clocks:
        time.sleep(0.3)
        t_wall = time.perf_counter()
        e0, e1 = timed(g_step.replay, 1)
        torch.cuda.synchronize()
        t_wall = time.perf_counter() - t_wall
    shard.barrier(info)
    step_ms = e0.elapsed_time(e1)
    # each stage alone, K launches in one graph, for the per-kernel launch durations
    pre_ev = timed(g_pre.replay, 1)
    cmb_ev = timed(g_cmb.replay, 1)
    # the same steps launched one call at a time from Python
    sl_ev = timed(step, args.steps)
    torch.cuda.synchronize()
    stage_ms = [pre_ev[0].elapsed_time(pre_ev[1]) / args.steps,
                cmb_ev[0].elapsed_time(cmb_ev[1]) / args.steps]
    stream_launch_ms = sl_ev[0].elapsed_time(sl_ev[1]) / args.steps
    del g_step, g_pre, g_cmb
    combine_ms = stage_ms[1]
    step_ms_max = shard.max_over_ranks(step_ms, info)
    ms_per_step = step_ms_max / args.steps

    # algorithmic bytes
    b_route, b_nq, b_cmb = bytes_per_token(H, E, k)
    idx_h = synth.host(case.row_idx)
    valid_slots = int(((idx_h >= 0) & (idx_h < case.R)).sum())
    cmb_bytes_nominal = T * b_cmb
    cmb_bytes_net = valid_slots * 2 * H + T * (8 * k + 2 * H)
    step_bytes_nominal = T * (b_route + b_nq + b_cmb)
    peak, peak_kind = measured_peaks()
    achieved_cmb = cmb_bytes_net / (combine_ms * 1e-3) / 1e9

    disp = None if args.no_dispatch else run_dispatch(eb, ids, E, dev, reps=max(5, min(args.steps, 200)))
    dec = None if args.no_decode else run_decode(eb, dev, reps=max(5, min(args.steps, 100)))
    far = None if args.no_finalize_ar else run_finalize_ar(eb, dev, peak, reps=max(5, min(args.steps, 100)))
    legs = {}
    if not args.no_legs:
        for name in ("large_e", "wide_topk"):
            legs[name] = run_leg(eb, name, dev, steps=max(5, min(args.steps, 50)), warmup=args.warmup, peak=peak)
            torch.cuda.empty_cache()

    # end to end through the same calls with host buffers (pinned), copies inside
    e2e = None if args.no_e2e else run_e2e(eb, case, dev, stream, ids, w, packed, sf, out,
                                           pre_expert, steps=max(3, min(args.steps, 8)))

    tokens_per_s = shard.weak_scaling_throughput(T, ms_per_step, info)
    result = None
    if rank == 0:
        cpu = None
        near = None
        if world == 1 and not args.no_cpu_baseline and T >= 512:
            n_sample = 512
            tokens, ch = host_sample(case, n_sample, seed=2)
            v, cores, reps, med = time_oracle(ch, tokens)
            cpu = {"value": v, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                   "sample": f"{n_sample} of 8192 tokens (all three stages), median of {reps} "
                             f"runs of {med:.2f} s"}
            near = near_threshold_report(case, packed, sf)
        clk = clocks.summary()
        result = {
            "metric": METRIC, "value": tokens_per_s, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": prefill_config(case, world),
            "hbm": {"step_bytes_nominal": step_bytes_nominal,
                    "step_gbs": step_bytes_nominal / (ms_per_step * 1e-3) / 1e9,
                    "frac_of_8tbs": step_bytes_nominal / (ms_per_step * 1e-3) / 1e9 / NOMINAL_HBM_GBS,
                    "frac_of_measured": step_bytes_nominal / (ms_per_step * 1e-3) / 1e9 / peak},
            "roofline": {"kernel": "combine", "bound": "hbm", "achieved": achieved_cmb,
                         "peak": peak, "peak_kind": peak_kind, "unit": "GB/s",
                         "frac": achieved_cmb / peak, "traffic": combine_traffic(cmb_bytes_net),
                         "traffic_source": "ncu, one combine launch at 2048 tokens, scaled by algorithmic bytes",
                         "bytes_per_launch": cmb_bytes_net,
                         "bytes_per_launch_nominal": cmb_bytes_nominal,
                         "avg_launch_ms": combine_ms},
            "stages_ms": {"route_norm_quant": stage_ms[0], "combine": stage_ms[1],
                          "how": "each stage alone, K launches in one CUDA graph, replayed between two events"},
            "stream_launch": {"ms_per_step": stream_launch_ms,
                              "tokens_per_s": shard.weak_scaling_throughput(T, stream_launch_ms, info),
                              "how": "the same K steps launched call by call from Python between two events"},
            "timing": "K steps captured in one CUDA graph, replayed between two events on the launching stream",
            "cpu_baseline": cpu,
            "e2e": e2e,
            "dispatch": disp,
            "decode": dec,
            "finalize_allreduce": far,
            "large_e": legs.get("large_e"),
            "wide_topk": legs.get("wide_topk"),
            "near_threshold": near,
            "gpu_launches": (pre_kernels + 1) * args.steps,
            "clocks": {"sm_mhz": clk["sm_mhz"], "sm_max_mhz": clk["sm_max_mhz"],
                       "reasons": clk["reasons"], "samples": clk["samples"],
                       "mem_mhz": clk.get("mem_mhz"), "power_w_max": clk.get("power_w_max"),
                       "power_limit_w": clk.get("power_limit_w"),
                       "timed_wall_s": t_wall},
        }
        print(json.dumps(result), flush=True)
    if eb.device_status() != 0:
        raise RuntimeError("a kernel reported a wait timeout")
    return result


def capture_graph(fn, n, dev):
    """n calls of fn captured in one CUDA graph (after one call on a side
    stream, which configures the kernels outside the capture)."""
    side = torch.cuda.Stream(dev)
    side.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(side):
        fn()
    torch.cuda.current_stream(dev).wait_stream(side)
    torch.cuda.synchronize(dev)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for _ in range(n):
            fn()
    return g


def run_dispatch(eb, ids, E, dev, reps):
    """The dispatch step (expert-grouped rows of this step's routing ids),
    timed apart from the step in CUDA-graph replays, so the time is the
    kernels' and not the Python binding's."""
    T, k = ids.shape
    off = torch.empty(E + 1, dtype=torch.int32, device=dev)
    idx = torch.empty(T, k, dtype=torch.int32, device=dev)
    tok = torch.empty(T * k, dtype=torch.int32, device=dev)
    ws = torch.empty(max(1, eb.dispatch_workspace_size(T, k, E)), dtype=torch.uint8, device=dev)
    us = _graph_us(lambda: eb.moe_dispatch(ids, E, 0, off, idx, tok, ws), reps, dev)
    n = T * k
    tiles = (n + 4095) // 4096    # 4096 entries per tile; the column scan runs above 32 tiles
    kernels = 1 if tiles <= 1 else (2 if tiles <= 32 else 3)
    return {"us": us, "entries": n, "experts": E, "kernels": kernels,
            "bytes": 12 * n, "gbs": 12 * n / (us * 1e-6) / 1e9,
            "bound": "latency", "how": f"{reps} calls per CUDA graph, one replay between two events",
            "valid_rows": int(off[-1].item())}


def _graph_us(fn, reps, dev):
    """Microseconds per call of `fn`: `reps` calls captured in one CUDA graph,
    replayed once between two events (launch-latency-sized work)."""
    side = torch.cuda.Stream(dev)
    side.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(side):
        for _ in range(3):
            fn()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for _ in range(reps):
            fn()
    g.replay()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record()
    g.replay()
    t1.record()
    torch.cuda.synchronize()
    del g
    return t0.elapsed_time(t1) * 1e3 / reps


def run_decode(eb, dev, reps):
    """The decode workload (128 tokens, H=8192, E=256, k=8, the gated residual
    join and next prenorm fused into the combine): latency of each stage and
    of the whole boundary, from CUDA-graph replays."""
    from expert_combine_b200 import synth
    case = synth.make_case("decode", device=dev, seed=synth.SEEDS["decode"])
    T, H, k = case.T, case.H, case.k
    ids = torch.empty(T, k, dtype=torch.int32, device=dev)
    w = torch.empty(T, k, dtype=torch.float32, device=dev)
    packed = torch.empty(T, H // 2, dtype=torch.uint8, device=dev)
    sf = torch.empty(T, H // 16, dtype=torch.uint8, device=dev)
    out = torch.empty(T, H, dtype=torch.bfloat16, device=dev)
    nxt = torch.empty(T, H, dtype=torch.bfloat16, device=dev)
    res = case.residual.clone()

    def route():
        eb.moe_route(case.logits, case.bias, case.mask, k, ids, w)

    def nq():
        eb.norm_quant_nvfp4(case.x, T, case.norm_w, case.gc, case.eps, case.gs, packed=packed, sf=sf)

    def pre():
        # the joint call: at this size the router runs beside the norm-quant
        eb.moe_route_norm_quant(case.logits, case.bias, case.mask, k, case.x, case.norm_w, case.gc,
                                case.eps, case.gs, topk_ids=ids, topk_weights=w, packed=packed, sf=sf)

    def cj():
        eb.expert_combine_join(case.expert_out, case.R, case.row_idx, w, case.post_w, case.post_gc,
                               case.eps, res, case.gain, case.alpha, case.beta, case.eps, case.next_w,
                               case.next_gc, case.eps, out=out, next_prenorm=nxt)

    def step():
        pre()
        cj()

    # router projection producing this step's logits: x [T, H] BF16, W [E, H] FP32 (seeded)
    g = torch.Generator(device="cpu")
    g.manual_seed(synth.SEEDS["decode"] + 7)
    w_router = (torch.randn(case.E, H, generator=g) / H ** 0.5).to(dev)
    w3_router = eb.router_weight_prepare(w_router)   # once, when the weight loads
    logits = torch.empty(T, case.E, dtype=torch.float32, device=dev)

    def proj():
        eb.router_logits(case.x, w3_router, 1.0, logits=logits)

    r = {"workload": f"decode T={T} H={H} E={case.E} k={k}, join + next prenorm fused",
         "router_logits_us": _graph_us(proj, reps, dev),
         "router_logits_bytes": case.E * H * 6 + T * H * 2 + T * case.E * 4,
         "route_us": _graph_us(route, reps, dev), "norm_quant_us": _graph_us(nq, reps, dev),
         "route_norm_quant_us": _graph_us(pre, reps, dev),
         "combine_join_us": _graph_us(cj, reps, dev), "step_us": _graph_us(step, reps, dev),
         "how": f"{reps} calls per CUDA graph, one replay between two events"}
    r["tokens_per_s"] = T / (r["step_us"] * 1e-6)
    return r


def run_finalize_ar(eb, dev, peak, reps):
    """The expert finalize fused with the tensor-parallel all-reduce at the
    pages' decode size (128 tokens of width 8192, top-8 of 256 experts split
    over 4 ranks), all four ranks' kernels in one launch on this GPU, each
    with its own workspace: on one device the peers' partials are read from
    local HBM, so the number measures the kernel, not NVLink."""
    from expert_combine_b200 import synth
    world, T, H, k, E = 4, 128, 8192, 8, 256
    c = synth.make_ep_case(T, H, k, E, world, seed=synth.SEEDS["decode"] + 11, device=dev)
    n = eb.finalize_ar_workspace_size(world, T, H)
    ws = [torch.empty(n, dtype=torch.uint8, device=dev) for _ in range(world)]
    for w in ws:
        eb.finalize_ar_workspace_init(w, world, T, H)
    outs = [torch.empty(T, H, dtype=torch.bfloat16, device=dev) for _ in range(world)]

    def call():
        eb.expert_finalize_allreduce_local(c.expert_out, c.R, c.row_idx, [c.weights] * world, c.norm_w, c.gc,
                                           c.eps, ws, T, outs=outs)

    us = _graph_us(call, reps, dev)
    rows = sum(c.R)
    # bytes of the one launch: every rank reads its rows, writes its partial,
    # reads all ranks' partials, writes its output; indices and weights
    hbm = rows * 2 * H + world * (T * H * 4 + world * T * H * 4 + T * H * 2 + T * k * 8)
    gbs = hbm / (us * 1e-6) / 1e9
    return {"workload": f"T={T} H={H} E={E} k={k}, experts split over {world} ranks, one-device exchange",
            "us": us, "bytes": hbm, "gbs": gbs, "frac_of_measured_hbm": gbs / peak, "bound": "hbm",
            "nvlink_bytes_per_rank": (world - 1) * T * H * 4,
            "how": f"{reps} calls per CUDA graph, one replay between two events"}


def run_leg(eb, name, dev, steps, warmup, peak):
    """Another workload of the pages at its full size, as one step per
    iteration: moe_route_norm_quant, then (wide top-k) the dispatch of the
    router's ids, then expert_combine with the router's weights.  The step's
    time (K back-to-back steps between two events) and each stage alone (K
    back-to-back launches), against the algorithmic bytes of each stage."""
    from expert_combine_b200 import synth
    case = synth.make_case(name, device=dev, seed=synth.SEEDS[name])
    T, H, E, k = case.T, case.H, case.E, case.k
    ids = torch.empty(T, k, dtype=torch.int32, device=dev)
    w = torch.empty(T, k, dtype=torch.float32, device=dev)
    packed = torch.empty(T, H // 2, dtype=torch.uint8, device=dev)
    sf = torch.empty(T, H // 16, dtype=torch.uint8, device=dev)
    out = torch.empty(T, H, dtype=torch.bfloat16, device=dev)
    chained = name == "wide_topk"          # stages end to end: the combine reads the dispatched rows
    if chained:
        offs = torch.empty(E + 1, dtype=torch.int32, device=dev)
        row_idx = torch.empty(T, k, dtype=torch.int32, device=dev)
        row_tok = torch.empty(T * k, dtype=torch.int32, device=dev)
        ws = torch.empty(max(16, eb.dispatch_workspace_size(T, k, E)), dtype=torch.uint8, device=dev)
    else:
        row_idx = case.row_idx
    stream = torch.cuda.current_stream(dev)

    def route():
        eb.moe_route(case.logits, case.bias, case.mask, k, ids, w)

    def norm_quant():
        eb.norm_quant_nvfp4(case.x, T, case.norm_w, case.gc, case.eps, case.gs, tp=case.tp, packed=packed, sf=sf)

    def pre():
        eb.moe_route_norm_quant(case.logits, case.bias, case.mask, k, case.x, case.norm_w, case.gc, case.eps,
                                case.gs, tp=case.tp, topk_ids=ids, topk_weights=w, packed=packed, sf=sf)

    def dispatch():
        eb.moe_dispatch(ids, E, 0, offs, row_idx, row_tok, ws)

    def combine():
        eb.expert_combine(case.expert_out, case.R, row_idx, w, case.post_w, case.post_gc, case.eps, out=out)

    def step():
        pre()
        if chained:
            dispatch()
        combine()

    def per_call_ms(fn, n):
        g = capture_graph(fn, n, dev)
        g.replay()
        torch.cuda.synchronize()
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        g.replay()
        t1.record(stream)
        torch.cuda.synchronize()
        del g
        return t0.elapsed_time(t1) / n

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    step_ms = per_call_ms(step, steps)
    stages = {"route": route, "norm_quant": norm_quant, "route_norm_quant": pre}
    if chained:
        stages["dispatch"] = dispatch
    stages["combine"] = combine
    stage_us = {key: per_call_ms(fn, steps) * 1e3 for key, fn in stages.items()}
    if eb.device_status() != 0:
        raise RuntimeError(f"{name}: a kernel reported a wait timeout")

    b_route, b_nq, b_cmb = bytes_per_token(H, E, k)
    idx_h = synth.host(row_idx)
    valid_slots = int(((idx_h >= 0) & (idx_h < case.R)).sum())
    bytes_ = {"route": T * b_route, "norm_quant": T * b_nq, "route_norm_quant": T * (b_route + b_nq),
              "dispatch": 12 * T * k,
              "combine": valid_slots * 2 * H + T * (8 * k + 2 * H)}
    stage_rep = {}
    for key, us in stage_us.items():
        gbs = bytes_[key] / (us * 1e-6) / 1e9
        stage_rep[key] = {"us": us, "bytes": bytes_[key], "gbs": gbs, "frac_of_measured_hbm": gbs / peak}
    step_bytes = T * (b_route + b_nq + b_cmb)
    step_gbs = step_bytes / (step_ms * 1e-3) / 1e9
    layout = f"rank-block [{case.tp}, {T}, {H // case.tp}]" if case.tp > 1 else "contiguous"
    return {"workload": f"{name} T={T} H={H} E={E} k={k}, norm-quant input {layout}"
                        + (", route -> dispatch -> combine end to end" if chained else ""),
            "tokens_per_s": T / (step_ms * 1e-3), "ms_per_step": step_ms,
            "step_bytes_nominal": step_bytes, "bytes_per_token": b_route + b_nq + b_cmb,
            "step_gbs": step_gbs, "frac_of_8tbs": step_gbs / NOMINAL_HBM_GBS, "frac_of_measured": step_gbs / peak,
            "stages": stage_rep, "valid_slots": valid_slots,
            "how": f"{steps} steps in one CUDA graph replayed between two events; each stage alone the same way",
            "gpu_launches_per_step": (eb.route_norm_quant_kernels(T, H, E, k, tp=case.tp)
                                      + (1 if not chained else 1 + (1 if T * k <= 4096 else
                                                                    (2 if T * k <= 32 * 4096 else 3))))}


def run_e2e(eb, case, dev, stream, ids, w, packed, sf, out, pre_expert, steps):
    """Host inputs (pinned) -> device -> the boundary's calls -> host outputs,
    every step, through the public API.  Steps are pipelined over three
    streams with two device buffer sets: step i's host-to-device copies run
    while step i - 1 computes and step i - 2's results come back (the copy
    engines work both directions at once).  The timed region holds all K steps'
    copies and calls, from the first copy in to the last copy out."""
    T, H, k = case.T, case.H, case.k
    names_in = (("logits", case.logits), ("mask", case.mask), ("x", case.x), ("expert", case.expert_out),
                ("idx", case.row_idx))
    h_in = {name: t.detach().cpu().pin_memory() for name, t in names_in}
    d_in = [{name: t for name, t in names_in}, {name: torch.empty_like(t) for name, t in names_in}]
    names_out = (("ids", ids), ("w", w), ("packed", packed), ("sf", sf), ("out", out))
    d_out = [{name: t for name, t in names_out}, {name: torch.empty_like(t) for name, t in names_out}]
    h_out = [{name: torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for name, t in names_out}
             for _ in range(2)]
    h2d = sum(t.numel() * t.element_size() for t in h_in.values())
    d2h = sum(t.numel() * t.element_size() for t in h_out[0].values())
    s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)

    def compute(b):
        i_, o_ = d_in[b], d_out[b]
        eb.moe_route_norm_quant(i_["logits"], case.bias, i_["mask"], k, i_["x"], case.norm_w, case.gc, case.eps,
                                case.gs, topk_ids=o_["ids"], topk_weights=o_["w"], packed=o_["packed"],
                                sf=o_["sf"])
        eb.expert_combine(i_["expert"], case.R, i_["idx"], o_["w"], case.post_w, case.post_gc, case.eps,
                          out=o_["out"])

    def run(n, t0=None, t1=None):
        ev = lambda: torch.cuda.Event()
        in_done, cmp_done, out_done = [ev() for _ in range(n)], [ev() for _ in range(n)], [ev() for _ in range(n)]
        s_in.wait_stream(stream)
        if t0 is not None:
            t0.record(s_in)
        for i in range(n):
            b = i % 2
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(cmp_done[i - 2])        # the set's previous step has read its inputs
                for name, h in h_in.items():
                    d_in[b][name].copy_(h, non_blocking=True)
                in_done[i].record(s_in)
            stream.wait_event(in_done[i])
            if i >= 2:
                stream.wait_event(out_done[i - 2])          # the set's previous results are on the host
            with torch.cuda.stream(stream):
                compute(b)
                cmp_done[i].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(cmp_done[i])
                for name, d in d_out[b].items():
                    h_out[b][name].copy_(d, non_blocking=True)
                out_done[i].record(s_out)
        stream.wait_stream(s_out)
        stream.wait_stream(s_in)
        if t1 is not None:
            t1.record(stream)

    run(2)
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    run(steps, s, e)
    torch.cuda.synchronize()
    ms = s.elapsed_time(e) / steps
    # the results match the device-resident step's (same inputs, same calls)
    for name, d in d_out[0].items():
        if not torch.equal(h_out[(steps - 1) % 2][name], d.cpu()):
            raise RuntimeError(f"e2e: host copy of {name} differs from the device result")
    return {"value": T / (ms * 1e-3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "ms_per_step": ms, "steps": steps,
            "how": "K steps pipelined over 3 streams and 2 device buffer sets, events around all of them"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--tokens", type=int, default=None,
                    help="tokens per rank (default: the workload's 8192); smaller for profiling")
    ap.add_argument("--no-decode", action="store_true",
                    help="skip the separate latency of the decode-sized boundary")
    ap.add_argument("--no-dispatch", action="store_true",
                    help="skip the separate timing of the dispatch step")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer end-to-end leg")
    ap.add_argument("--no-legs", action="store_true",
                    help="skip the large-E gate and wide top-k workloads")
    ap.add_argument("--no-finalize-ar", action="store_true",
                    help="skip the separate timing of the finalize + all-reduce (one-device exchange)")
    ap.add_argument("--separate", action="store_true",
                    help="issue moe_route and norm_quant_nvfp4 as two calls instead of moe_route_norm_quant")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--nvtx", action="store_true",
                    help="NVTX ranges around every library call (for a profiler's timeline)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    # the reference arm runs on rank 0 alone and joins no process group
    info = shard.init("nccl") if args.impl == "ours" else shard.rank_info()
    try:
        if args.impl == "reference":
            return run_reference(args, info)
        import contextlib

        import expert_combine_b200 as eb
        with eb.trace() if args.nvtx else contextlib.nullcontext():
            run_ours(args, info)
        return 0
    finally:
        if args.impl == "ours":
            shard.finalize(info)


if __name__ == "__main__":
    sys.exit(main())
