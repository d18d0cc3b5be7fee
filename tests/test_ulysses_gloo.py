"""Sequence-parallel (Ulysses) attention on gloo ranks (CPU): the product's
``ulysses_attention`` runs its real exchanges (all-reduce MAX of the three
amax values, the all-to-all of the codes and the return all-to-all of the
output) through ``TorchComm`` over gloo, with the oracle standing in for each
rank's kernels (a context whose amax, ring and cast are the oracle's, and the
oracle's attention and a torch permute in place of the attention and regroup
kernels).  Every rank's output, ring and scales must equal one pass over the
whole sequence on one process.

vLLM-Omni docs, "Quantized KV Cache", Configuration: the offline diffusion
example shards the DiT over a Ulysses degree of 4.  vLLM docs, "FP8 ViT
encoder attention", usage: the per-tensor amax is a max over the whole
tensor, so each rank needs the other ranks' maxima."""
import os
import queue
import socket
import time

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

H, D = 4, 128
S_TOTAL = 320          # 2.5 key tiles of 128: a ragged last tile
STATIC_VALUES = (6.0, 5.5, 7.25)
PLAN = [("dyn", 0), ("dyn", 1), ("static", 2), ("skip", 3), ("dyn", 4)]


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _inputs(p):
    import synthetic
    q, k, v, cu = synthetic.small_qkv(900 + p, [S_TOTAL], H=H, scale=1.0 + 0.75 * p)
    q = q.clone()
    q[:, H - 1, 9] *= 6.0          # one head group holds the largest |q|
    if p == 4:
        k = k.clone()
        k[S_TOTAL - 1, 0, 0] = float("inf")   # non-finite amax: not pushed
    return q, k, v


def _oracle_kernels(qar):
    """Stand-ins for the attention and regroup kernels (this process only)."""
    import oracle
    import synthetic

    def varlen_fwd(q8, k8, v8, cu, max_seqlen, descale, softmax_scale=0.0, p_rule=1,
                   schedule=qar.SCHED_AUTO):
        # the oracle evaluates each row whole; every schedule computes that rule
        rule = oracle.P_EXP2 if p_rule == qar.P_EXP2 else oracle.P_LINEAR_LOG
        return torch.from_numpy(oracle.attention_fp8(q8.numpy(), k8.numpy(), v8.numpy(),
                                                     np.asarray(cu), descale, rule=rule))

    def varlen_fwd_bf16(q, k, v, cu, max_seqlen, softmax_scale=0.0):
        b = [synthetic.bf16_bits(x) for x in (q, k, v)]
        return torch.from_numpy(oracle.attention_bf16(b[0], b[1], b[2], np.asarray(cu)))

    def regroup_heads(x, groups, to_groups=True):
        if to_groups:
            T, Hh, Dd = x.shape
            return x.view(T, groups, Hh // groups, Dd).permute(1, 0, 2, 3).contiguous()
        G, T, Hn, Dd = x.shape
        return x.permute(1, 0, 2, 3).reshape(T, G * Hn, Dd).contiguous()

    qar.varlen_fwd = varlen_fwd
    qar.varlen_fwd_bf16 = varlen_fwd_bf16
    qar.regroup_heads = regroup_heads


def _worker(rank, world, port, out_q):
    import sys
    here = os.path.dirname(os.path.abspath(__file__))
    sys.path[:0] = [os.path.dirname(here), here]
    import quantization_amax_reduce_b200 as qar
    _oracle_kernels(qar)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from oracle_context import OracleContext
        ctx = OracleContext(STATIC_VALUES)
        comm = qar.TorchComm()
        assert comm.size() == world and comm.rank() == rank
        S_loc = S_TOTAL // world
        mine = slice(rank * S_loc, (rank + 1) * S_loc)
        results = []
        for kind, p in PLAN:
            q, k, v = _inputs(p)
            mode = {"dyn": qar.DYNAMIC, "static": qar.STATIC, "skip": qar.SKIP}[kind]
            o = qar.ulysses_attention(ctx, 0, mode, q[mine].contiguous(), k[mine].contiguous(),
                                      v[mine].contiguous(), comm=comm)
            results.append((o.numpy().copy(), [float(d) for d in ctx.ds],
                            [r.slots.tolist() for r in ctx.rings]))
        out_q.put((rank, results))
    finally:
        dist.destroy_process_group()


def _reference():
    """The same passes on the whole sequence in one process, oracle only."""
    import oracle
    import synthetic
    rings = [oracle.Ring() for _ in range(3)]
    cu = np.array([0, S_TOTAL], dtype=np.int32)
    ref = []
    for kind, p in PLAN:
        q, k, v = _inputs(p)
        bits = [synthetic.bf16_bits(x) for x in (q, k, v)]
        if kind == "skip":
            out = oracle.attention_bf16(bits[0], bits[1], bits[2], cu)
            ds = None
        else:
            codes, ds = [], []
            for t in range(3):
                if kind == "dyn":
                    a, nf = oracle.amax(bits[t], cu, H, D)
                    qs, d = rings[t].dynamic_step(a, nf)
                else:
                    qs, d = oracle.scales_from_bound(np.float32(STATIC_VALUES[t]))
                codes.append(oracle.quantize(bits[t], cu, H, D, qs))
                ds.append(float(d))
            out = oracle.attention_fp8(codes[0], codes[1], codes[2], cu, ds)
        ref.append((out, ds, [r.slots.tolist() for r in rings]))
    return ref


@pytest.mark.parametrize("world", [2, 4])
def test_ulysses_ranks_equal_one_pass_over_the_whole_sequence(world):
    port = _free_port()
    ctx = mp.get_context("spawn")
    out_q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, out_q)) for r in range(world)]
    for p in procs:
        p.start()
    got = {}
    deadline = time.monotonic() + 300
    try:
        while len(got) < world:
            try:
                rank, res = out_q.get(timeout=2)
                got[rank] = res
            except queue.Empty:
                dead = [p.exitcode for p in procs if p.exitcode not in (None, 0)]
                assert not dead, f"a rank failed: exit codes {dead}"
                assert time.monotonic() < deadline, "ranks did not report in time"
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    for p in procs:
        assert p.exitcode == 0
    ref = _reference()
    S_loc = S_TOTAL // world
    for i, (kind, p) in enumerate(PLAN):
        want, ds, slots = ref[i]
        for rank in range(world):
            o, g_ds, g_slots = got[rank][i]
            w = want[rank * S_loc:(rank + 1) * S_loc]
            np.testing.assert_array_equal(o, w, err_msg=f"{kind} pass {p} rank {rank}")
            if ds is not None:
                assert g_ds == ds, (kind, p, rank)
            assert g_slots == slots, (kind, p, rank)


class _FakeComm:
    def __init__(self, n):
        self.n = n

    def size(self):
        return self.n

    def rank(self):
        return 0


def test_argument_checks_before_any_exchange():
    import quantization_amax_reduce_b200 as qar
    x = torch.zeros(8, 4, D, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="multiple of the number of ranks"):
        qar.ulysses_attention(None, 0, qar.DYNAMIC, x, x, x, comm=_FakeComm(3))
    with pytest.raises(ValueError, match="mode"):
        qar.ulysses_attention(None, 0, qar.RING, x, x, x, comm=_FakeComm(2))
    with pytest.raises(ValueError, match="same shape"):
        qar.ulysses_attention(None, 0, qar.DYNAMIC, x, x[:4], x, comm=_FakeComm(2))
    with pytest.raises(ValueError, match="head_dim"):
        y = torch.zeros(8, 4, 64, dtype=torch.bfloat16)
        qar.ulysses_attention(None, 0, qar.DYNAMIC, y, y, y, comm=_FakeComm(2))
