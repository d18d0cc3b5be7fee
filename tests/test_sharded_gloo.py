"""Head-sharded dynamic quantisation on two gloo ranks (CPU), with the oracle
standing in for each rank's kernels: the per-tensor amax is the only value
that crosses ranks (an all-reduce MAX of three floats), after which every
rank's ring, scales and codes equal those of one pass over all heads.

vLLM docs, "FP8 ViT encoder attention", usage: scales come from a ring of
observed Q/K/V amax values; the amax is a max over the whole tensor, so a
rank that holds some of the heads needs the other ranks' maxima."""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

H, D = 8, 128
LENS = [37, 130, 5]
PASSES = 4


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _inputs(p):
    """bf16 bit patterns [T, H, D] for pass p, with one large channel on a
    head of the second shard so the shards' amax differ."""
    import synthetic
    q, k, v, cu = synthetic.small_qkv(500 + p, LENS, H=H, scale=1.0 + p)
    out = []
    for x in (q, k, v):
        x = x.clone()
        x[:, H - 1, 3] *= 8.0
        out.append(synthetic.bf16_bits(x))
    return out, cu


def _worker(rank, world, port, q):
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import oracle
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        hs = H // world
        heads = slice(rank * hs, (rank + 1) * hs)
        rings = [oracle.Ring() for _ in range(3)]
        results = []
        for p in range(PASSES):
            bits, cu = _inputs(p)
            shard = [np.ascontiguousarray(b[:, heads, :]) for b in bits]
            local = torch.tensor([oracle.amax(x, cu, hs, D)[0] for x in shard], dtype=torch.float32)
            dist.all_reduce(local, op=dist.ReduceOp.MAX)
            codes, scales = [], []
            for t in range(3):
                qs, ds = rings[t].dynamic_step(float(local[t]), False)
                scales.append((float(qs), float(ds)))
                codes.append(oracle.quantize(shard[t], cu, hs, D, qs))
            results.append((scales, [c.tobytes() for c in codes], [r.slots.tolist() for r in rings]))
        q.put((rank, results))
    finally:
        dist.destroy_process_group()


def test_two_rank_head_sharded_pass_equals_the_unsharded_pass():
    import oracle
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    import queue
    import time
    got = {}
    deadline = time.monotonic() + 300
    while len(got) < world:
        try:
            rank, res = q.get(timeout=2)
            got[rank] = res
        except queue.Empty:
            dead = [p.exitcode for p in procs if p.exitcode not in (None, 0)]
            assert not dead, f"a rank failed: exit codes {dead}"
            assert time.monotonic() < deadline, "ranks did not report in time"
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    # the same passes on all heads in one process
    rings = [oracle.Ring() for _ in range(3)]
    hs = H // world
    for p in range(PASSES):
        bits, cu = _inputs(p)
        for t in range(3):
            a, nf = oracle.amax(bits[t], cu, H, D)
            qs, ds = rings[t].dynamic_step(a, nf)
            full = oracle.quantize(bits[t], cu, H, D, qs)
            for rank in range(world):
                scales, codes, slots = got[rank][p]
                assert scales[t] == (float(qs), float(ds)), (p, t, rank)
                want = np.ascontiguousarray(full[:, rank * hs:(rank + 1) * hs, :]).tobytes()
                assert codes[t] == want, (p, t, rank)
                assert slots[t] == rings[t].slots.tolist(), (p, t, rank)
