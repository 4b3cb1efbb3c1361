"""Collective set-up of the expert finalize + tensor-parallel all-reduce.

TensorRT-LLM PR 21356, description, "Fused finalize + all-reduce": with the
experts split over the ranks of one node, the expert finalize and the TP
all-reduce run as one kernel, a one-shot exchange through peer memory.  Its
workspace is built collectively -- every rank either ends with every peer's
workspace mapped or raises the same error -- and released so that no rank
frees memory a peer may still map.

One process per GPU; the process group (NCCL on GPUs, gloo in the CPU tests)
carries only the set-up messages.  The exchange itself is the kernel's
(``expert_finalize_allreduce`` in the C library).  The peer-memory operations
are an object with alloc / init / handle / open / close / free, CUDA IPC by
default; the CPU tests pass a stand-in.
"""
from __future__ import annotations

from typing import Optional

import torch

from . import _lib


class FinalizeAllReduceError(RuntimeError):
    """Raised on every rank, with the same message, when the collective set-up fails."""


class CudaIpcOps:
    """Peer memory through CUDA IPC: a whole cudaMalloc allocation per rank."""

    def size(self, world: int, T_max: int, H: int) -> int:
        return _lib.finalize_ar_workspace_size(world, T_max, H)

    def alloc(self, nbytes: int) -> int:
        return _lib.ipc_alloc(nbytes)

    def init(self, ptr: int, world: int, T_max: int, H: int) -> None:
        _lib.finalize_ar_workspace_init(ptr, world, T_max, H)
        torch.cuda.synchronize()

    def handle(self, ptr: int) -> bytes:
        return _lib.ipc_get_handle(ptr)

    def open(self, handle: bytes) -> int:
        return _lib.ipc_open(handle)

    def close(self, ptr: int) -> None:
        _lib.ipc_close(ptr)

    def free(self, ptr: int) -> None:
        _lib.ipc_free(ptr)

    def quiesce(self) -> None:
        torch.cuda.synchronize()


def _dist():
    import torch.distributed as dist
    return dist


def _all_ok(items, what: str) -> None:
    errors = [(r, e) for r, e in enumerate(items) if e]
    if errors:
        raise FinalizeAllReduceError(f"finalize all-reduce {what} failed: " +
                                     "; ".join(f"rank {r}: {e}" for r, e in errors))


class FinalizeAllReduce:
    """One rank's share of the exchange: its own workspace and its mappings
    of every peer's, for batches of up to ``T_max`` tokens of width ``H``.

    Construction is a collective over ``group``: every rank allocates and
    initialises its workspace, the handles are exchanged, every rank maps
    every peer's; a failure anywhere makes every rank release what it holds
    and raise the same FinalizeAllReduceError.
    """

    def __init__(self, T_max: int, H: int, group=None, ops=None):
        dist = _dist()
        self.ops = ops if ops is not None else CudaIpcOps()
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        self.T_max, self.H = int(T_max), int(H)
        self.local: Optional[int] = None
        self.peers: list = []
        self._closed = False

        # 1. own workspace and its handle
        err, handle = None, None
        try:
            nbytes = self.ops.size(self.world, self.T_max, self.H)
            if nbytes == 0:
                raise ValueError(f"unsupported sizes (world={self.world}, T_max={self.T_max}, H={self.H})")
            self.local = self.ops.alloc(nbytes)
            self.ops.init(self.local, self.world, self.T_max, self.H)
            handle = self.ops.handle(self.local)
        except Exception as exc:   # reported to every rank below
            err = f"{type(exc).__name__}: {exc}"
        gathered = [None] * self.world
        dist.all_gather_object(gathered, (err, handle), group=group)
        try:
            _all_ok([g[0] for g in gathered], "workspace allocation")
        except FinalizeAllReduceError:
            self._free_local()
            raise

        # 2. every peer's workspace mapped here
        opened, err = {}, None
        for q in range(self.world):
            if q == self.rank:
                continue
            try:
                opened[q] = self.ops.open(gathered[q][1])
            except Exception as exc:
                err = f"mapping rank {q}'s workspace: {type(exc).__name__}: {exc}"
                break
        errs = [None] * self.world
        dist.all_gather_object(errs, err, group=group)
        try:
            _all_ok(errs, "peer mapping")
        except FinalizeAllReduceError:
            for ptr in opened.values():
                self.ops.close(ptr)
            dist.barrier(group=group)      # every peer has unmapped this rank's workspace
            self._free_local()
            raise
        self.peers = [self.local if q == self.rank else opened[q] for q in range(self.world)]

    def _free_local(self) -> None:
        if self.local is not None:
            self.ops.free(self.local)
            self.local = None

    def __call__(self, expert_out: torch.Tensor, num_rows: int, row_idx: torch.Tensor, weights: torch.Tensor,
                 norm_w: torch.Tensor, gain_center: float, eps: float, out: Optional[torch.Tensor] = None,
                 stream=None) -> torch.Tensor:
        """This rank's call; every rank makes the same sequence of calls."""
        if self._closed:
            raise FinalizeAllReduceError("the finalize all-reduce workspace has been released")
        return _lib.expert_finalize_allreduce(expert_out, num_rows, row_idx, weights, norm_w, gain_center, eps,
                                              self.peers, self.rank, self.T_max, out=out, stream=stream)

    def close(self) -> None:
        """Collective release: unmap the peers' workspaces, then -- once every
        rank has unmapped this one -- free it.  Calling it again does nothing."""
        if self._closed:
            return
        dist = _dist()
        self._closed = True
        if hasattr(self.ops, "quiesce"):
            self.ops.quiesce()             # this rank's calls have finished
        dist.barrier(group=self.group)     # ... and every peer's
        for q, ptr in enumerate(self.peers):
            if q != self.rank:
                self.ops.close(ptr)
        dist.barrier(group=self.group)     # nobody maps this rank's workspace any more
        self._free_local()
        self.peers = []
