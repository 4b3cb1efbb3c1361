"""Build libmoe_boundary.so in-tree with nvcc for sm_100a (no JIT, no torch)."""
from __future__ import annotations

import os
import shutil
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libmoe_boundary.so")
SOURCES = ["moe_boundary.cu", "api.cu", "combine.cu", "norm_quant.cu", "route.cu", "decode.cu", "router_proj.cu", "dispatch.cu",
           "dispatch_noalloc.cu", "finalize_ar.cu",
           "common.cuh", "ring.cuh", "route.cuh", "internal.h", "tmap.h"]
HEADER = os.path.join(os.path.dirname(HERE), "include", "moe_boundary.h")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "--fmad=false",               # no contraction: the arithmetic order is part of the contract
    "-Xcompiler", "-fPIC", "-shared",
]


def nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA library cannot be built")


def _inputs():
    return [os.path.join(CSRC, s) for s in SOURCES] + [HEADER]


def is_stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(p) > t for p in _inputs())


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile the library if it is missing or older than its sources."""
    if not force and not is_stale():
        return LIB
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = [nvcc(), *NVCC_FLAGS, "-I", os.path.dirname(HEADER), os.path.join(CSRC, "moe_boundary.cu"),
           "-o", tmp]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    import sys
    print(build(force=True, verbose="-v" in sys.argv))
