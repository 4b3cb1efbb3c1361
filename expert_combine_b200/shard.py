"""Host-side plumbing for running the boundary on several GPUs, one process per
GPU (torch.distributed; NCCL on GPUs, gloo for the CPU tests).

The boundary is per token: tokens shard across GPUs with no exchange on the
data path.  A rank either processes its own batch (weak scaling, the
benchmark) or a contiguous range of a global batch (``shard_range``).  The
collectives here are only for timing: a barrier around the timed region and the
maximum of the ranks' times.
"""
from __future__ import annotations

import datetime
import os
from dataclasses import dataclass

import torch


@dataclass(frozen=True)
class RankInfo:
    world: int
    rank: int
    local: int


def rank_info() -> RankInfo:
    """World size, rank and local rank from the launcher's environment."""
    return RankInfo(int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
                    int(os.environ.get("LOCAL_RANK", "0")))


def init(backend: str = "nccl", timeout_s: float = 120.0) -> RankInfo:
    """Join the process group when the world has more than one rank (a short
    timeout, so ranks that wait for a missing peer end with an error)."""
    info = rank_info()
    if info.world > 1:
        import torch.distributed as dist
        kw = {}
        if backend == "nccl":
            torch.cuda.set_device(info.local)
            kw["device_id"] = torch.device("cuda", info.local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s), **kw)
    return info


def finalize(info: RankInfo) -> None:
    if info.world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def barrier(info: RankInfo) -> None:
    if info.world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, info: RankInfo) -> float:
    """The largest of the ranks' values (the timed region ends when the slowest
    rank does)."""
    if info.world == 1:
        return float(x)
    import torch.distributed as dist
    dev = torch.device("cuda", torch.cuda.current_device()) if dist.get_backend() == "nccl" else torch.device("cpu")
    t = torch.tensor([float(x)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def shard_range(total: int, info: RankInfo) -> tuple[int, int]:
    """Contiguous [begin, end) of ``total`` tokens for this rank: every token
    on exactly one rank, range sizes differing by at most one."""
    base, extra = divmod(total, info.world)
    begin = info.rank * base + min(info.rank, extra)
    return begin, begin + base + (1 if info.rank < extra else 0)


def rank_seed(base_seed: int, info: RankInfo) -> int:
    """Seed of this rank's synthetic batch (weak scaling: distinct batches)."""
    return base_seed + info.rank


def weak_scaling_throughput(units_per_rank: int, max_ms_per_step: float, info: RankInfo) -> float:
    """Units per second of the whole job: every rank's units over the slowest
    rank's time."""
    return units_per_rank * info.world / (max_ms_per_step * 1e-3)
