"""GPU parity of the fused quantisation kernel and the device ring against
the oracle: FP8 codes, scales and ring state must match bit for bit.

vLLM docs, "FP8 ViT encoder attention": on-the-fly Q/K/V quantisation with a
16-entry amax ring (usage section), static scales (scale file format
section), quant launches plus unpadding (notes)."""
import numpy as np
import pytest
import torch

import oracle
import synthetic
import quantization_amax_reduce_b200 as qar
from tests.parity import (OracleLayer, assert_codes_equal, assert_ring_equal,
                          assert_scales_equal, bits)

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _cast_inputs():
    hi = (np.arange(1 << 16, dtype=np.uint32) << 16)
    lows = np.array([0x0000, 0x0001, 0x7FFF, 0x8000, 0x8001, 0xFFFF, 0x4000, 0xC000,
                     0x1234, 0xFEDC], dtype=np.uint32)
    grid = (hi[:, None] | lows[None, :]).reshape(-1)
    rng = np.random.Generator(np.random.PCG64(11))
    rnd = rng.integers(0, 1 << 32, size=1 << 22, dtype=np.uint64).astype(np.uint32)
    # every midpoint between adjacent E4M3 values and its fp32 neighbours,
    # at several scales so the products land on ties
    pos = oracle.e4m3_value(np.arange(0x7F, dtype=np.uint8))
    mids = ((pos[:-1] + pos[1:]) / 2).astype(np.float32)
    mid_bits = np.concatenate([mids.view(np.uint32), mids.view(np.uint32) + 1,
                               mids.view(np.uint32) - 1])
    mid_bits = np.concatenate([mid_bits, mid_bits | 0x80000000])
    return np.concatenate([grid, rnd, mid_bits]).view(np.float32)


def test_cast_matches_oracle_on_bit_patterns():
    x = _cast_inputs()
    got = qar.e4m3_encode(torch.from_numpy(x).to(DEV), 1.0).cpu().numpy()
    want = oracle.e4m3_encode(x)
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, [(hex(x.view(np.uint32)[i]), hex(got[i]), hex(want[i])) for i in bad[:5]]


@pytest.mark.parametrize("scale", [448.0 / 210.0, 0.37, 3.0e4])
def test_cast_with_scale_matches_oracle(scale):
    x = (np.arange(1 << 16, dtype=np.uint32) << 16).view(np.float32)
    got = qar.e4m3_encode(torch.from_numpy(x).to(DEV), scale).cpu().numpy()
    with np.errstate(over="ignore", invalid="ignore"):
        y = x * np.float32(scale)
    np.testing.assert_array_equal(got, oracle.e4m3_encode(y))


def _gpu(t):
    return t.to(DEV)


def test_c1_dynamic_first_pass_bit_exact():
    q, k, v, cu = synthetic.qkv(1)
    ctx = qar.Context(1)
    cu_d = torch.as_tensor(cu, device=DEV)
    q8, k8, v8 = ctx.quantize_qkv(0, qar.DYNAMIC, _gpu(q), _gpu(k), _gpu(v), cu_d, 256)
    ol = OracleLayer()
    want = ol.dynamic_pass([bits(q), bits(k), bits(v)], cu, 2)
    for g, w, n in zip((q8, k8, v8), want, "qkv"):
        assert_codes_equal(g, w, n)
    assert_scales_equal(ctx, 0, ol)
    assert_ring_equal(ctx, 0, ol)
    assert ctx.get_error() == 0


def test_c3_static_page_values_bit_exact():
    q, k, v, cu = synthetic.qkv(3)
    ctx = qar.Context(1)
    ctx.set_static_scales(0, 224.0, 198.0, 210.0)
    cu_d = torch.as_tensor(cu, device=DEV)
    q8, k8, v8 = ctx.quantize_qkv(0, qar.STATIC, _gpu(q), _gpu(k), _gpu(v), cu_d, 8192)
    ol = OracleLayer()
    ol.set_static((224.0, 198.0, 210.0))
    want = ol.static_pass([bits(q), bits(k), bits(v)], cu, 16)
    for g, w, n in zip((q8, k8, v8), want, "qkv"):
        assert_codes_equal(g, w, n)
    qs, ds = ctx.get_scales(0)
    assert ds[0] == 0.5 and qs[0] == 2.0 and ds[2] == 0.46875
    assert_scales_equal(ctx, 0, ol)
    # static passes never touch the ring
    slots, meta = ctx.get_ring_state(0)
    assert (meta[:, 1] == 0).all()


def test_c2_sixteen_dynamic_passes_ring_and_codes():
    w = synthetic.WORKLOADS[2]
    ctx = qar.Context(1)
    ol = OracleLayer()
    cu = w.cu_seqlens(0)
    cu_d = torch.as_tensor(cu, device=DEV)
    max_len = int(np.diff(cu).max())
    for p in range(w.passes):
        q, k, v, _ = synthetic.qkv(2, 0, p, device=DEV)
        q8, k8, v8 = ctx.quantize_qkv(0, qar.DYNAMIC, q, k, v, cu_d, max_len)
        want = ol.dynamic_pass([bits(q), bits(k), bits(v)], cu, w.H)
        assert_scales_equal(ctx, 0, ol)
        assert_ring_equal(ctx, 0, ol)
        if p in (0, 1, w.passes - 1):
            for g, ww, n in zip((q8, k8, v8), want, "qkv"):
                assert_codes_equal(g, ww, f"pass {p} {n}")
    assert ctx.get_error() == 0


def _pad(x, cu, S_max, fill):
    B = len(cu) - 1
    T, H, D = x.shape
    out = torch.full((B, S_max, H, D), fill, dtype=x.dtype, device=x.device)
    for b in range(B):
        out[b, :cu[b + 1] - cu[b]] = x[cu[b]:cu[b + 1]]
    return out


def test_unpad_from_padded_source_bit_exact():
    lens = [300, 1, 129, 0, 77]
    q, k, v, cu = synthetic.small_qkv(21, lens, H=3, scale=4.0, device=DEV)
    S_max = 320
    big = 3.0e38   # padding that would dominate the amax if it leaked in
    pq, pk, pv = (_pad(t, cu, S_max, big) for t in (q, k, v))
    start = torch.arange(len(lens), dtype=torch.int32, device=DEV) * S_max
    ctx = qar.Context(2)
    cu_d = torch.as_tensor(cu, device=DEV)
    T = int(cu[-1])
    q8, k8, v8 = ctx.quantize_qkv(1, qar.DYNAMIC, pq, pk, pv, cu_d, S_max, total_tokens=T,
                                  src_seq_start=start)
    ol = OracleLayer()
    want = ol.dynamic_pass([bits(q), bits(k), bits(v)], cu, 3)
    for g, w, n in zip((q8, k8, v8), want, "qkv"):
        assert_codes_equal(g, w, n)
    assert_scales_equal(ctx, 1, ol)


def test_interleaved_qkv_source_bit_exact():
    q, k, v, cu = synthetic.small_qkv(22, [200, 57], H=4, device=DEV)
    qkv = torch.stack([q, k, v], dim=1).contiguous()     # [T, 3, H, D]
    ctx = qar.Context(1)
    cu_d = torch.as_tensor(cu, device=DEV)
    q8, k8, v8 = ctx.quantize_qkv(0, qar.DYNAMIC, qkv[:, 0], qkv[:, 1], qkv[:, 2], cu_d, 200)
    ol = OracleLayer()
    want = ol.dynamic_pass([bits(q), bits(k), bits(v)], cu, 4)
    for g, w, n in zip((q8, k8, v8), want, "qkv"):
        assert_codes_equal(g, w, n)


def test_nan_ignored_and_inf_reported():
    q, k, v, cu = synthetic.small_qkv(23, [64, 64], H=2, device=DEV)
    q[3, 1, 5] = float("nan")
    k[70, 0, 0] = float("inf")
    ctx = qar.Context(1)
    cu_d = torch.as_tensor(cu, device=DEV)
    q8, k8, v8 = ctx.quantize_qkv(0, qar.DYNAMIC, q, k, v, cu_d, 64)
    ol = OracleLayer()
    want = ol.dynamic_pass([bits(q), bits(k), bits(v)], cu, 2)
    for g, w, n in zip((q8, k8, v8), want, "qkv"):
        assert_codes_equal(g, w, n)
    assert q8[3, 1, 5].item() == 0x7F
    assert_scales_equal(ctx, 0, ol)
    assert_ring_equal(ctx, 0, ol)
    slots, meta = ctx.get_ring_state(0)
    assert meta[1, 1] == 0              # the infinite K amax was not pushed
    assert ctx.get_error() == 5         # FP8ATTN_ERR_NONFINITE
    assert ctx.get_error() == 0         # cleared


def test_bad_cu_seqlens_reported_and_nothing_written():
    q, k, v, cu = synthetic.small_qkv(24, [10, 20], H=1, device=DEV)
    ctx = qar.Context(1)
    bad = torch.tensor([0, 25, 30], dtype=torch.int32, device=DEV)   # length 25 > max 20
    outs = [torch.full((30, 1, 128), 0xAB, dtype=torch.uint8, device=DEV) for _ in range(3)]
    ctx.quantize_qkv(0, qar.DYNAMIC, q, k, v, bad, 20, out=outs)
    assert ctx.get_error() == 6
    for o in outs:
        assert (o == 0xAB).all()
    slots, meta = ctx.get_ring_state(0)
    assert (meta[:, 1] == 0).all()


def test_static_without_scales_is_rejected():
    q, k, v, cu = synthetic.small_qkv(25, [8], H=1, device=DEV)
    ctx = qar.Context(1)
    with pytest.raises(qar.FP8AttnError):
        ctx.quantize_qkv(0, qar.STATIC, q, k, v, torch.as_tensor(cu, device=DEV), 8)


def test_standalone_ring_update_and_export():
    ctx = qar.Context(3)
    ol = [OracleLayer() for _ in range(3)]
    rng = np.random.Generator(np.random.PCG64(5))
    for step in range(21):
        for layer in range(3):
            a = rng.uniform(0.5, 40.0, size=3).astype(np.float32)
            ctx.amax_ring_update(layer, torch.from_numpy(a).to(DEV))
            for t in range(3):
                ol[layer].qs[t], ol[layer].ds[t] = ol[layer].rings[t].dynamic_step(a[t])
    for layer in range(3):
        assert_ring_equal(ctx, layer, ol[layer])
        assert_scales_equal(ctx, layer, ol[layer])
    exp = ctx.export_static_scales(1.5)
    for layer in range(3):
        for t in range(3):
            assert exp[layer, t] == ol[layer].rings[t].export_value(1.5)


def test_ring_state_save_and_resume():
    ctx = qar.Context(1)
    for a in ([1.0, 2.0, 3.0], [5.0, 0.5, 7.0], [2.0, 9.0, 1.0]):
        ctx.amax_ring_update(0, torch.tensor(a, device=DEV))
    slots, meta = ctx.get_ring_state(0)
    scales = ctx.get_scales(0)
    ctx2 = qar.Context(1)
    ctx2.set_ring_state(0, slots, meta)
    s2, m2 = ctx2.get_ring_state(0)
    np.testing.assert_array_equal(s2, slots)
    np.testing.assert_array_equal(m2, meta)
    np.testing.assert_array_equal(ctx2.get_scales(0)[0], scales[0])
    np.testing.assert_array_equal(ctx2.get_scales(0)[1], scales[1])


def test_dynamic_passes_capture_in_a_cuda_graph():
    """Device-resident ring state: 16 quantisation passes captured once and
    replayed give the same ring, scales and codes as 16 eager passes."""
    lens = [700, 333]
    H = 4
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    cu_d = torch.as_tensor(cu, device=DEV)
    T = int(cu[-1])
    inputs = [synthetic.small_qkv(100 + p, lens, H=H, scale=1.0 + p, device=DEV)[:3]
              for p in range(16)]
    eager = qar.Context(1)
    for q, k, v in inputs:
        e8 = eager.quantize_qkv(0, qar.DYNAMIC, q, k, v, cu_d, 700)
    graphed = qar.Context(1)
    src = [torch.empty_like(inputs[0][i]) for i in range(3)]
    outs = [torch.empty((T, H, 128), dtype=torch.uint8, device=DEV) for _ in range(3)]
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            graphed.quantize_qkv(0, qar.DYNAMIC, src[0], src[1], src[2], cu_d, 700, out=outs,
                                 stream=s)
    torch.cuda.current_stream().wait_stream(s)
    for q, k, v in inputs:
        for d, x in zip(src, (q, k, v)):
            d.copy_(x)
        g.replay()
    torch.cuda.synchronize()
    a_slots, a_meta = eager.get_ring_state(0)
    b_slots, b_meta = graphed.get_ring_state(0)
    np.testing.assert_array_equal(a_slots, b_slots)
    np.testing.assert_array_equal(a_meta, b_meta)
    for x, y in zip(e8, outs):
        assert torch.equal(x, y)
