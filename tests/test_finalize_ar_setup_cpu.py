"""Collective set-up and release of the finalize all-reduce's peer
workspaces (expert_combine_b200.finalize_ar) on 2 and 3 CPU ranks with the
gloo backend and a stand-in for the peer-memory operations: every rank ends
with every peer's workspace mapped, or every rank raises the same error and
releases what it holds; on release no rank frees its workspace before every
peer has unmapped it (TensorRT-LLM PR 21356, "Fused finalize + all-reduce":
construction is collective, release never frees memory a peer may still
map)."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class FakeOps:
    """Peer memory stand-in: addresses are (rank, serial) pairs encoded as ints;
    a handle names the owner's address.  Every operation is logged."""

    def __init__(self, rank, fail=None):
        self.rank, self.fail, self.log, self.serial = rank, fail or {}, [], 0

    def _maybe_fail(self, op):
        if self.fail.get(op) == self.rank:
            raise RuntimeError(f"injected {op} failure")

    def size(self, world, T_max, H):
        return 256 + 8 * world * T_max + 8 * T_max * H

    def alloc(self, nbytes):
        self._maybe_fail("alloc")
        self.serial += 1
        ptr = 1000 * (self.rank + 1) + self.serial
        self.log.append(("alloc", ptr))
        return ptr

    def init(self, ptr, world, T_max, H):
        self._maybe_fail("init")
        self.log.append(("init", ptr))

    def handle(self, ptr):
        return ptr.to_bytes(8, "little") + bytes(56)

    def open(self, handle):
        self._maybe_fail("open")
        owner_ptr = int.from_bytes(handle[:8], "little")
        mapped = 10 ** 6 + owner_ptr
        self.log.append(("open", mapped))
        return mapped

    def close(self, ptr):
        self.log.append(("close", ptr))

    def free(self, ptr):
        self.log.append(("free", ptr))


def _worker(rank, world, port, fail, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world), RANK=str(rank),
                      LOCAL_RANK=str(rank))
    try:
        from expert_combine_b200 import shard
        from expert_combine_b200.finalize_ar import FinalizeAllReduce, FinalizeAllReduceError
        info = shard.init("gloo", timeout_s=60)
        ops = FakeOps(rank, fail)
        result = {"rank": rank}
        try:
            far = FinalizeAllReduce(128, 8192, ops=ops)
            result["peers"] = list(far.peers)
            result["local"] = far.local
            far.close()
            far.close()                       # a second release does nothing
            result["closed_peers"] = far.peers
        except FinalizeAllReduceError as exc:
            result["error"] = str(exc)
        result["log"] = ops.log
        shard.barrier(info)
        shard.finalize(info)
        q.put(result)
    except Exception as exc:
        q.put({"rank": rank, "crash": repr(exc)})


def _run(world, fail=None):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, fail, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(world):
        r = q.get(timeout=120)
        res[r["rank"]] = r
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r in res.values():
        assert "crash" not in r, r
    return res


@pytest.mark.parametrize("world", [2, 3])
def test_every_rank_maps_every_peer(world):
    res = _run(world)
    locals_ = {r: res[r]["local"] for r in range(world)}
    for r in range(world):
        peers = res[r]["peers"]
        assert len(peers) == world and peers[r] == locals_[r]
        for q in range(world):
            if q != r:
                assert peers[q] == 10 ** 6 + locals_[q]     # rank q's workspace, mapped here
        log = res[r]["log"]
        # release: unmap every peer, then free the own workspace, once
        closes = [i for i, (op, _) in enumerate(log) if op == "close"]
        frees = [i for i, (op, _) in enumerate(log) if op == "free"]
        assert len(closes) == world - 1 and len(frees) == 1 and max(closes) < frees[0]
        assert log[frees[0]][1] == locals_[r]
        assert res[r]["closed_peers"] == []


@pytest.mark.parametrize("op,bad", [("alloc", 1), ("init", 0), ("open", 1)])
def test_a_failure_on_one_rank_fails_every_rank_alike(op, bad):
    world = 3
    res = _run(world, {op: bad})
    msgs = {res[r].get("error") for r in range(world)}
    assert len(msgs) == 1 and None not in msgs          # the same error everywhere
    msg = msgs.pop()
    assert f"rank {bad}" in msg and f"injected {op} failure" in msg
    for r in range(world):
        log = res[r]["log"]
        allocs = [p for o, p in log if o == "alloc"]
        frees = [p for o, p in log if o == "free"]
        assert sorted(allocs) == sorted(frees)            # whatever was allocated is freed
        opens = [p for o, p in log if o == "open"]
        closes = [p for o, p in log if o == "close"]
        assert sorted(opens) == sorted(closes)            # whatever was mapped is unmapped
        if frees and closes:
            last_close = max(i for i, (o, _) in enumerate(log) if o == "close")
            first_free = min(i for i, (o, _) in enumerate(log) if o == "free")
            assert last_close < first_free
