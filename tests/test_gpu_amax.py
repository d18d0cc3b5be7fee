"""The amax-only entry point (fp8attn_amax_qkv) against the oracle: a max of
|x| over the valid tokens of each of Q, K and V, NaN ignored, with no cast and
no change to any ring or scale.

vLLM docs, "FP8 ViT encoder attention", usage: the dynamic scales come from
the amax of the whole tensor, pushed into a 16-entry ring."""
import numpy as np
import pytest
import torch

import oracle
import synthetic
import quantization_amax_reduce_b200 as qar

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _want(x, cu, H, **kw):
    a, nf = oracle.amax(synthetic.bf16_bits(x), cu, H, 128, **kw)
    return float("inf") if nf else float(np.float32(a))


def _check(got, ts, cu, H, tag, **kw):
    g = got.cpu().numpy()
    for i, t in enumerate(ts):
        w = _want(t, cu, H, **kw)
        assert (np.isinf(g[i]) if np.isinf(w) else g[i] == np.float32(w)), (tag, i, g[i], w)


def test_padded_source_ignores_the_padding():
    lens = [300, 1, 129, 0, 77]
    H = 3
    q, k, v, cu = synthetic.small_qkv(31, lens, H=H, scale=3.0, device=DEV)
    S_max = 320
    B = len(lens)

    def pad(x):
        out = torch.full((B, S_max, H, 128), 3.0e38, dtype=x.dtype, device=DEV)
        for b in range(B):
            out[b, :lens[b]] = x[cu[b]:cu[b + 1]]
        return out

    start = torch.arange(B, dtype=torch.int32, device=DEV) * S_max
    ctx = qar.Context(1)
    got = ctx.amax_qkv(pad(q), pad(k), pad(v), torch.as_tensor(cu, device=DEV), S_max,
                       total_tokens=int(cu[-1]), src_seq_start=start)
    _check(got, (q, k, v), cu, H, "padded")


def test_no_ring_or_scale_changes_and_repeat_calls_start_clean():
    lens = [513, 64]
    H = 4
    cu_d = None
    ctx = qar.Context(2)
    ring0 = [ctx.get_ring_state(l) for l in range(2)]
    scales0 = [ctx.get_scales(l) for l in range(2)]
    # a large amax, then a small one: the second call must not see the first's
    for i, scale in enumerate((1000.0, 0.01, 5.0)):
        q, k, v, cu = synthetic.small_qkv(40 + i, lens, H=H, scale=scale, device=DEV)
        cu_d = torch.as_tensor(cu, device=DEV)
        got = ctx.amax_qkv(q, k, v, cu_d, max(lens))
        torch.cuda.synchronize()
        _check(got, (q, k, v), cu, H, f"call {i}")
    for l in range(2):
        s, m = ctx.get_ring_state(l)
        np.testing.assert_array_equal(s, ring0[l][0])
        np.testing.assert_array_equal(m, ring0[l][1])
        for a, b in zip(ctx.get_scales(l), scales0[l]):
            np.testing.assert_array_equal(a, b)


def test_nan_is_ignored_and_inf_is_reported():
    lens = [200, 33]
    H = 2
    q, k, v, cu = synthetic.small_qkv(50, lens, H=H, scale=1.0, device=DEV)
    q[7, 1, 3] = float("nan")          # NaN: not a candidate for the max
    k[210, 0, 100] = float("-inf")     # -inf: |x| is infinite
    v[0, 0, 0] = float("nan")
    v[1, 1, 1] = 1.0e30
    ctx = qar.Context(1)
    got = ctx.amax_qkv(q, k, v, torch.as_tensor(cu, device=DEV), max(lens))
    torch.cuda.synchronize()
    g = got.cpu().numpy()
    assert np.isfinite(g[0]) and np.isinf(g[1]) and g[2] == np.float32(torch.tensor(
        1.0e30, dtype=torch.bfloat16).float().item())
    _check(got, (q, k, v), cu, H, "nonfinite")


def test_all_empty_batch_is_zero():
    ctx = qar.Context(1)
    cu = np.zeros(4, dtype=np.int32)
    x = torch.zeros(1, 2, 128, dtype=torch.bfloat16, device=DEV)
    got = ctx.amax_qkv(x, x, x, torch.as_tensor(cu, device=DEV), 16, total_tokens=0)
    torch.cuda.synchronize()
    assert got.cpu().tolist() == [0.0, 0.0, 0.0]


@pytest.mark.parametrize("cid", [2, 4])
def test_full_size_workloads(cid):
    """The varlen outlier workload (3 sequences of 1024..8192, 16 heads) and the
    single 32760-token, 40-head sequence, in the launch shape the dynamic
    quantisation uses."""
    q, k, v, cu = synthetic.qkv(cid, device=DEV)
    H = q.shape[1]
    ctx = qar.Context(1)
    got = ctx.amax_qkv(q, k, v, torch.as_tensor(cu, device=DEV), int(np.diff(cu).max()))
    torch.cuda.synchronize()
    _check(got, (q, k, v), cu, H, f"workload {cid}")
