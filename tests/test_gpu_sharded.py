"""The head-sharded dynamic pass through the C ABI on one GPU: two contexts
stand in for two ranks, each holding half of the heads (strided views, no
copies); the all-reduce MAX of the three amax values is a torch.maximum on
the device.  Codes, scales and rings must equal one fused DYNAMIC pass over
all heads, pass after pass, including a pass whose amax is infinite.

vLLM docs, "FP8 ViT encoder attention", usage: scales come from a ring of
observed Q/K/V amax values, a max over the whole tensor."""
import numpy as np
import pytest
import torch

import oracle
import synthetic
import quantization_amax_reduce_b200 as qar

pytestmark = pytest.mark.gpu

DEV = "cuda"


def test_two_shard_pass_equals_the_fused_pass():
    lens = [700, 129, 333]
    H = 8
    hs = H // 2
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    cu_d = torch.as_tensor(cu, device=DEV)
    full_ctx = qar.Context(1)
    shard_ctx = [qar.Context(1), qar.Context(1)]
    for p in range(6):
        q, k, v, _ = synthetic.small_qkv(600 + p, lens, H=H, scale=1.0 + 0.5 * p, device=DEV)
        q[:, H - 1, 5] *= 10.0                 # the shards' amax differ
        if p == 4:
            k[3, 1, 7] = float("inf")          # non-finite amax: reported, not pushed
        want = full_ctx.quantize_qkv(0, qar.DYNAMIC, q, k, v, cu_d, max(lens))
        shards = [tuple(x[:, i * hs:(i + 1) * hs, :] for x in (q, k, v)) for i in range(2)]
        amax = [shard_ctx[i].amax_qkv(*shards[i], cu_d, max(lens)) for i in range(2)]
        # the amax of a shard is the oracle's
        for i in range(2):
            for t in range(3):
                bits = synthetic.bf16_bits(shards[i][t].contiguous())
                a, nf = oracle.amax(bits, cu, hs, 128)
                got = float(amax[i][t].item())
                assert (np.isinf(got) if nf else got == float(np.float32(a))), (p, i, t)
        reduced = torch.maximum(amax[0], amax[1])      # the all-reduce MAX
        got = []
        for i in range(2):
            shard_ctx[i].amax_ring_update(0, reduced)
            got.append(shard_ctx[i].quantize_qkv(0, qar.RING, *shards[i], cu_d, max(lens)))
        torch.cuda.synchronize()
        for t in range(3):
            assert torch.equal(torch.cat([got[0][t], got[1][t]], dim=1), want[t]), (p, t)
        ws, wm = full_ctx.get_ring_state(0)
        for i in range(2):
            gs, gm = shard_ctx[i].get_ring_state(0)
            np.testing.assert_array_equal(gs, ws)
            np.testing.assert_array_equal(gm, wm)
            for a, b in zip(shard_ctx[i].get_scales(0), full_ctx.get_scales(0)):
                np.testing.assert_array_equal(a, b)
        # a non-finite amax is reported on both paths
        e_full = full_ctx.get_error()
        e_shard = [c.get_error() for c in shard_ctx]
        assert (e_full != 0) == (p == 4) and all((e != 0) == (p == 4) for e in e_shard), \
            (p, e_full, e_shard)


def test_helper_without_a_process_group_is_one_dynamic_pass():
    lens = [300, 17]
    q, k, v, cu = synthetic.small_qkv(77, lens, H=4, scale=2.0, device=DEV)
    cu_d = torch.as_tensor(cu, device=DEV)
    a, b = qar.Context(1), qar.Context(1)
    want = a.quantize_qkv(0, qar.DYNAMIC, q, k, v, cu_d, max(lens))
    got = qar.head_sharded_dynamic_quantize(b, 0, q, k, v, cu_d, max(lens))
    torch.cuda.synchronize()
    for x, y in zip(got, want):
        assert torch.equal(x, y)
    np.testing.assert_array_equal(a.get_ring_state(0)[0], b.get_ring_state(0)[0])
