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
