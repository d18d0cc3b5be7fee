"""bench.py's multi-rank host logic on two gloo ranks (CPU): the timed value
is the max over ranks, the throughput aggregates every rank's units over that
time, and the reference arm runs on rank 0 only."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        r, w, lr = bench.dist_env()
        slowest = bench.max_over_ranks(1.0 + rank, dist, torch.device("cpu"))
        agg = bench.aggregate_throughput(100.0, w, slowest)
        # the reference arm does nothing on ranks other than 0
        ref_rc = bench.run_reference(bench.parse_args(["--impl", "reference", "--steps", "1",
                                                        "--warmup", "0"])) if rank != 0 else 0
        q.put((rank, r, w, slowest, agg, ref_rc))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_weak_scaling_aggregate():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=5) for _ in range(world))
    for rank, r, w, slowest, agg, ref_rc in res:
        assert r == rank and w == world
        assert slowest == 2.0                 # max of 1.0 and 2.0 on every rank
        assert agg == 100.0 * world / 2.0     # all ranks' units over the slowest time
        assert ref_rc == 0


def test_single_rank_identity():
    import bench
    assert bench.max_over_ranks(3.5, None) == 3.5
    assert bench.aggregate_throughput(10.0, 1, 2.0) == 5.0


def test_bench_starts_its_own_ranks_and_aggregates():
    """`python bench.py --gpus 2` without a torchrun environment starts two
    ranks itself; --dry-run replaces the GPU work by a CPU stand-in on gloo,
    so the launcher, the max-over-ranks time and the whole-job aggregate are
    checked here without a GPU."""
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = {k: v for k, v in os.environ.items()
           if k not in ("RANK", "WORLD_SIZE", "LOCAL_RANK", "MASTER_ADDR", "MASTER_PORT")}
    r = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--gpus", "2",
                        "--dry-run", "--steps", "5", "--warmup", "1"],
                       capture_output=True, text=True, timeout=300, env=env, cwd=root)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout            # rank 0 alone prints
    d = json.loads(lines[0])
    assert d["n_gpus"] == 2 and d["dry_run"] and d["steps"] == 5
    # whole-job throughput: both ranks' steps over the slowest rank's time
    slowest = d["ms_per_step"] * d["steps"] / 1e3
    assert abs(d["value"] - 2 * 5 / slowest) < 1e-6 * d["value"]
