"""The multi-GPU host plumbing (expert_combine_b200.shard) on two CPU ranks
with the gloo backend: process-group set-up from the launcher's environment,
the barrier, the maximum over ranks, token ranges and the weak-scaling
throughput.  No GPU and no data-path collective are involved: the boundary is
per token, so ranks only meet for timing."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world), RANK=str(rank),
                      LOCAL_RANK=str(rank))
    try:
        from expert_combine_b200 import shard
        info = shard.init("gloo", timeout_s=60)
        assert (info.world, info.rank) == (world, rank)
        shard.barrier(info)
        m = shard.max_over_ranks(10.0 + 3.0 * rank, info)
        ranges = [shard.shard_range(t, info) for t in (0, 1, 7, 8192, 8193)]
        seed = shard.rank_seed(1003, info)
        thr = shard.weak_scaling_throughput(8192, m, info)
        shard.barrier(info)
        shard.finalize(info)
        q.put((rank, m, ranges, seed, thr))
    except Exception as e:  # reported to the parent
        q.put((rank, repr(e), None, None, None))


@pytest.mark.parametrize("world", [2, 3])
def test_ranks_on_cpu(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(world):
        r = q.get(timeout=120)
        res[r[0]] = r
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    slowest = 10.0 + 3.0 * (world - 1)
    for r in range(world):
        _, m, ranges, seed, thr = res[r]
        assert m == slowest, m
        assert seed == 1003 + r
        assert thr == pytest.approx(8192 * world / (slowest * 1e-3))
    # every token on exactly one rank, sizes within one of each other
    for i, total in enumerate((0, 1, 7, 8192, 8193)):
        got = sorted(res[r][2][i] for r in range(world))
        assert got[0][0] == 0 and got[-1][1] == total
        for (a0, a1), (b0, b1) in zip(got, got[1:]):
            assert a1 == b0
        sizes = [b - a for a, b in got]
        assert max(sizes) - min(sizes) <= 1


def test_single_rank_needs_no_process_group(monkeypatch):
    from expert_combine_b200 import shard
    monkeypatch.delenv("WORLD_SIZE", raising=False)
    info = shard.init("gloo")
    assert info.world == 1
    assert shard.max_over_ranks(4.5, info) == 4.5
    assert shard.shard_range(10, info) == (0, 10)
    shard.barrier(info)
    shard.finalize(info)


def test_reference_arm_runs_on_rank_zero_only():
    """Under a two-rank launch the bench's reference arm (the oracle on the
    host cores) prints nothing and exits 0 on every rank but rank 0."""
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, WORLD_SIZE="2", RANK="1", LOCAL_RANK="1", MASTER_ADDR="127.0.0.1",
               MASTER_PORT=str(_free_port()))
    r = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--steps", "1", "--warmup", "3"], env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""


def test_reference_arm_json_line():
    """A single-process reference arm prints one JSON line with the contract's
    keys; its config names the same workload the CUDA arm reports (built by
    the same function from the same seeded batch)."""
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = {k: v for k, v in os.environ.items() if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK")}
    r = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference", "--tokens", "512",
                        "--steps", "1", "--warmup", "3"], env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["value"] > 0 and d["higher_is_better"] is True
    assert d["warmup"] >= 3 and d["steps"] == 1
    c = d["config"]
    assert c["workload"].startswith("prefill T=512 H=8192") and c["tokens_per_rank"] == 512
    assert 0 < c["valid_tokens"] <= 512 and 0 < c["valid_slots"] <= 512 * c["top_k"]
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]
