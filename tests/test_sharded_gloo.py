"""Head-sharded dynamic quantisation on two gloo ranks (CPU): the product's
``head_sharded_dynamic_quantize`` runs its real all-reduce (MAX of three
floats, through ``TorchComm`` over gloo) with the oracle standing in for each
rank's kernels.  After it every rank's ring, scales and codes equal those of
one pass over all heads.

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
    """bf16 [T, H, D] tensors for pass p, with one large channel on a head of
    the second shard so the shards' amax differ."""
    import synthetic
    q, k, v, cu = synthetic.small_qkv(500 + p, LENS, H=H, scale=1.0 + p)
    out = []
    for x in (q, k, v):
        x = x.clone()
        x[:, H - 1, 3] *= 8.0
        out.append(x)
    return out, cu


def _worker(rank, world, port, q):
    import sys
    here = os.path.dirname(os.path.abspath(__file__))
    sys.path[:0] = [os.path.dirname(here), here]
    import quantization_amax_reduce_b200 as qar
    from oracle_context import OracleContext
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        hs = H // world
        heads = slice(rank * hs, (rank + 1) * hs)
        ctx = OracleContext()
        results = []
        for p in range(PASSES):
            x, cu = _inputs(p)
            shard = [t[:, heads, :] for t in x]          # strided views, as on a GPU
            codes = qar.head_sharded_dynamic_quantize(ctx, 0, *shard, cu, max(LENS))
            scales = [(float(a), float(b)) for a, b in zip(ctx.qs, ctx.ds)]
            results.append((scales, [c.numpy().tobytes() for c in codes],
                            [r.slots.tolist() for r in ctx.rings]))
        q.put((rank, results))
    finally:
        dist.destroy_process_group()


def test_two_rank_head_sharded_pass_equals_the_unsharded_pass():
    import oracle
    import synthetic
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
        x, cu = _inputs(p)
        bits = [synthetic.bf16_bits(t) for t in x]
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
