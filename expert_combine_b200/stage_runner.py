"""Run one entry point of the library on a named synthetic workload, a few
times, and print its CUDA-graph time: the command line behind the profiler
summaries (one kernel, a handful of launches, a bounded device footprint).

  python -m expert_combine_b200.stage_runner STAGE WORKLOAD [--tokens T] [--reps N]

STAGE: route, norm_quant, route_norm_quant, combine, dispatch.
WORKLOAD: a name from synth.WORKLOADS (tiny, decode, prefill, large_e,
wide_topk); --tokens overrides its token count.
"""
from __future__ import annotations

import argparse
import statistics

import torch

from . import _lib as eb
from . import synth


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("stage", choices=["route", "norm_quant", "route_norm_quant", "combine", "dispatch"])
    ap.add_argument("workload", choices=sorted(synth.WORKLOADS))
    ap.add_argument("--tokens", type=int, default=None)
    ap.add_argument("--reps", type=int, default=3, help="eager calls before the timed graph")
    args = ap.parse_args(argv)
    dev = torch.device("cuda", torch.cuda.current_device())
    c = synth.make_case(args.workload, device=dev, T=args.tokens, join=False)
    T, H, E, k = c.T, c.H, c.E, c.k
    ids = torch.empty(T, k, dtype=torch.int32, device=dev)
    w = torch.empty(T, k, dtype=torch.float32, device=dev)
    eb.moe_route(c.logits, c.bias, c.mask, k, ids, w)
    packed = torch.empty(T, H // 2, dtype=torch.uint8, device=dev)
    sf = torch.empty(T, H // 16, dtype=torch.uint8, device=dev)
    out = torch.empty(T, H, dtype=torch.bfloat16, device=dev)
    offs = torch.empty(E + 1, dtype=torch.int32, device=dev)
    row_idx = torch.empty(T, k, dtype=torch.int32, device=dev)
    row_tok = torch.empty(T * k, dtype=torch.int32, device=dev)
    ws = torch.empty(max(16, eb.dispatch_workspace_size(T, k, E)), dtype=torch.uint8, device=dev)
    calls = {
        "route": lambda: eb.moe_route(c.logits, c.bias, c.mask, k, ids, w),
        "norm_quant": lambda: eb.norm_quant_nvfp4(c.x, T, c.norm_w, c.gc, c.eps, c.gs, tp=c.tp, packed=packed,
                                                  sf=sf),
        "route_norm_quant": lambda: eb.moe_route_norm_quant(c.logits, c.bias, c.mask, k, c.x, c.norm_w, c.gc,
                                                            c.eps, c.gs, tp=c.tp, topk_ids=ids, topk_weights=w,
                                                            packed=packed, sf=sf),
        "combine": lambda: eb.expert_combine(c.expert_out, c.R, c.row_idx, w, c.post_w, c.post_gc, c.eps, out=out),
        "dispatch": lambda: eb.moe_dispatch(ids, E, 0, offs, row_idx, row_tok, ws),
    }
    fn = calls[args.stage]
    for _ in range(args.reps):
        fn()
    torch.cuda.synchronize()
    n = 10
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for _ in range(n):
            fn()
    times = []
    for _ in range(5):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        g.replay()
        b.record()
        torch.cuda.synchronize()
        times.append(a.elapsed_time(b) * 1e3 / n)
    status = eb.device_status()
    print(f"{args.stage} {args.workload} T={T} H={H} E={E} k={k}: {statistics.median(times):.1f} us per call "
          f"(CUDA graph of {n}), status {status}")
    return 0 if status == 0 else 1


if __name__ == "__main__":
    raise SystemExit(main())
