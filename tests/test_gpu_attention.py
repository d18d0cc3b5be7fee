"""GPU parity of the tcgen05 varlen attention kernels against the oracle.

FP8: vLLM-Omni docs, "Quantized KV Cache", overview (quantised Q/K/V feed a
full, non-causal attention operator) and vLLM docs, "FP8 ViT encoder
attention" (per-tensor scales).  BF16: vLLM-Omni parameters table (skipped
layers keep the native dtype).  Tolerance: max |err| <= 1e-2 and mean |err|
<= 1e-3 against the oracle's fp64 attention with the same P rule."""
import math

import numpy as np
import pytest
import torch

import oracle
import synthetic
import quantization_amax_reduce_b200 as qar
from tests.parity import (OracleLayer, assert_attention_close, assert_codes_equal,
                          assert_ring_equal, assert_scales_equal, bits, sample_rows)

pytestmark = pytest.mark.gpu

DEV = "cuda"

# both P rules of the FP8 kernel, each against the oracle's statement of it
RULES = [pytest.param(qar.P_LINEAR_LOG, oracle.P_LINEAR_LOG, id="linear_log"),
         pytest.param(qar.P_EXP2, oracle.P_EXP2, id="exp2")]


def _codes(T, H, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(T, H, 128, generator=g) * scale
    return x.to(torch.float8_e4m3fn).view(torch.uint8)



CASES = [
    ([1], 1), ([5], 2), ([128], 1), ([129], 1), ([256], 2), ([257], 1), ([383], 3),
    ([1000, 17], 2), ([5, 300, 129], 3), ([64, 0, 200, 0], 2), ([513, 1, 255], 1),
    # enough (sequence, head, 256-query block) units to fill whole waves of
    # the GPU: ragged sequences through both the main and the tail kernel
    ([257, 1, 129], 60), ([1000, 17], 40),
]


@pytest.mark.parametrize("rule,orule", RULES)
@pytest.mark.parametrize("lens,H", CASES)
def test_fp8_attention_small_shapes(lens, H, rule, orule):
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    T = int(cu[-1])
    q8, k8, v8 = (_codes(T, H, s, 6.0) for s in (1, 2, 3))
    # v ~ N(0, 0.1^2): outputs of the size the workloads produce, so the
    # absolute tolerance measures the kernel rather than bf16 output rounding
    ds = torch.tensor([0.05, 0.04, 1.0 / 60.0], dtype=torch.float32)
    out = qar.varlen_fwd(q8.to(DEV), k8.to(DEV), v8.to(DEV), torch.as_tensor(cu, device=DEV),
                         max(lens), ds.to(DEV), p_rule=rule)
    want = oracle.attention_fp8(q8.numpy(), k8.numpy(), v8.numpy(), cu, ds.tolist(),
                                return_alternative=True, rule=orule)
    assert_attention_close(out, want, what=f"fp8 {lens} H={H} {orule}")


@pytest.mark.parametrize("lens,H", CASES[:8])
def test_bf16_attention_small_shapes(lens, H):
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    q, k, v, _ = synthetic.small_qkv(31, lens, H=H, scale=1.5)
    v = (v.float() * (1.0 / 15.0)).to(torch.bfloat16)   # v ~ N(0, 0.1^2)
    out = qar.varlen_fwd_bf16(q.to(DEV), k.to(DEV), v.to(DEV), torch.as_tensor(cu, device=DEV),
                              max(lens))
    want = oracle.attention_bf16(bits(q), bits(k), bits(v), cu)
    assert_attention_close(out, want, what=f"bf16 {lens} H={H}")


@pytest.mark.parametrize("rule,orule", RULES)
def test_sharp_softmax_rescales(rule, orule):
    """Large score range so the reference max moves across key tiles (O
    rescaling in TMEM) and many p fall in E4M3's subnormal range."""
    lens = [900]
    H = 2
    cu = np.array([0, 900], dtype=np.int32)
    g = torch.Generator().manual_seed(9)
    # increasing key norms along the sequence: later tiles hold larger maxima
    ramp = torch.linspace(0.2, 3.0, 900).view(900, 1, 1)
    q8 = (torch.randn(900, H, 128, generator=g) * 4).to(torch.float8_e4m3fn).view(torch.uint8)
    k8 = (torch.randn(900, H, 128, generator=g) * 4 * ramp).to(torch.float8_e4m3fn).view(torch.uint8)
    v8 = (torch.randn(900, H, 128, generator=g) * 4).to(torch.float8_e4m3fn).view(torch.uint8)
    ds = [0.25, 0.25, 0.025]
    out = qar.varlen_fwd(q8.to(DEV), k8.to(DEV), v8.to(DEV), torch.as_tensor(cu, device=DEV),
                         900, torch.tensor(ds, device=DEV), p_rule=rule)
    want = oracle.attention_fp8(q8.numpy(), k8.numpy(), v8.numpy(), cu, ds, return_alternative=True,
                                rule=orule)
    assert_attention_close(out, want, what=f"sharp {orule}")


@pytest.mark.parametrize("rule,orule", RULES)
def test_explicit_softmax_scale(rule, orule):
    cu = np.array([0, 300], dtype=np.int32)
    q8, k8, v8 = (_codes(300, 2, s, 3.0) for s in (4, 5, 6))
    ds = [0.1, 0.1, 0.05]
    out = qar.varlen_fwd(q8.to(DEV), k8.to(DEV), v8.to(DEV), torch.as_tensor(cu, device=DEV),
                         300, torch.tensor(ds, device=DEV), softmax_scale=0.3, p_rule=rule)
    want = oracle.attention_fp8(q8.numpy(), k8.numpy(), v8.numpy(), cu, ds, scale=0.3,
                                return_alternative=True, rule=orule)
    assert_attention_close(out, want, what=f"scale 0.3 {orule}")


@pytest.mark.parametrize("rule,orule", RULES)
def test_c1_end_to_end_through_the_boundary(rule, orule):
    q, k, v, cu = synthetic.qkv(1)
    ctx = qar.Context(1)
    cu_d = torch.as_tensor(cu, device=DEV)
    q8, k8, v8 = ctx.quantize_qkv(0, qar.DYNAMIC, q.to(DEV), k.to(DEV), v.to(DEV), cu_d, 256)
    out = qar.varlen_fwd(q8, k8, v8, cu_d, 256, ctx.descale_ptr(0), p_rule=rule)
    ol = OracleLayer()
    codes = ol.dynamic_pass([bits(q), bits(k), bits(v)], cu, 2)
    want = oracle.attention_fp8(*codes, cu, [float(x) for x in ol.ds], return_alternative=True,
                                rule=orule)
    # the error against unquantised fp64 attention on the bf16 inputs is reported
    ref = oracle.attention_bf16(bits(q), bits(k), bits(v), cu)
    assert_attention_close(out, want, what=f"c1 {orule}", unquantized=ref)


@pytest.mark.parametrize("rule,orule", RULES)
def test_c3_full_size_sampled_rows(rule, orule):
    """The benchmarked configuration: S=8192, 16 heads, static 224/198/210.
    The oracle quantises the bf16 inputs itself (codes and scales must equal
    the kernel's bit for bit) and attends on its own codes."""
    q, k, v, cu = synthetic.qkv(3, device=DEV)
    ctx = qar.Context(1)
    ctx.set_static_scales(0, 224.0, 198.0, 210.0)
    cu_d = torch.as_tensor(cu, device=DEV)
    q8, k8, v8 = ctx.quantize_qkv(0, qar.STATIC, q, k, v, cu_d, 8192)
    out = qar.varlen_fwd(q8, k8, v8, cu_d, 8192, ctx.descale_ptr(0), p_rule=rule)
    ol = OracleLayer()
    ol.set_static([224.0, 198.0, 210.0])
    hq, hk, hv = bits(q), bits(k), bits(v)
    codes = ol.static_pass([hq, hk, hv], cu, 16)
    for g, w, n in zip((q8, k8, v8), codes, "qkv"):
        assert_codes_equal(g, w, n)
    assert_scales_equal(ctx, 0, ol)
    rows = sample_rows(cu, 192, seed=3)
    want = oracle.attention_fp8(*codes, cu, [float(x) for x in ol.ds], rows=rows,
                                return_alternative=True, rule=orule)
    ref = oracle.attention_bf16(hq, hk, hv, cu, rows=rows)
    assert_attention_close(out, want, rows=rows, what=f"c3 {orule}", unquantized=ref)


@pytest.mark.parametrize("rule,orule", RULES)
def test_c2_varlen_after_sixteen_passes_sampled_rows(rule, orule):
    """Config 2 after its 16 dynamic passes: the oracle follows the ring
    through every pass, quantises the last pass itself and attends on its
    own codes."""
    w = synthetic.WORKLOADS[2]
    ctx = qar.Context(1)
    cu = w.cu_seqlens(0)
    cu_d = torch.as_tensor(cu, device=DEV)
    max_len = int(np.diff(cu).max())
    ol = OracleLayer()
    for p in range(w.passes):
        q, k, v, _ = synthetic.qkv(2, 0, p, device=DEV)
        q8, k8, v8 = ctx.quantize_qkv(0, qar.DYNAMIC, q, k, v, cu_d, max_len)
        hq, hk, hv = bits(q), bits(k), bits(v)
        if p == w.passes - 1:
            codes = ol.dynamic_pass([hq, hk, hv], cu, w.H)
        else:
            for t, x in enumerate((hq, hk, hv)):
                a, nf = oracle.amax(x, cu, w.H, 128)
                ol.qs[t], ol.ds[t] = ol.rings[t].dynamic_step(a, nf)
    for g, ww, n in zip((q8, k8, v8), codes, "qkv"):
        assert_codes_equal(g, ww, n)
    assert_scales_equal(ctx, 0, ol)
    assert_ring_equal(ctx, 0, ol)
    out = qar.varlen_fwd(q8, k8, v8, cu_d, max_len, ctx.descale_ptr(0), p_rule=rule)
    rows = sample_rows(cu, 128, seed=2)
    want = oracle.attention_fp8(*codes, cu, [float(x) for x in ol.ds], rows=rows,
                                return_alternative=True, rule=orule)
    ref = oracle.attention_bf16(hq, hk, hv, cu, rows=rows)
    assert_attention_close(out, want, rows=rows, what=f"c2 {orule}", unquantized=ref)


def _nan_boundary_case(kind):
    """Three sequences whose boundaries fall inside 128-key tiles; the
    sequence after each boundary holds non-finite values in its first rows,
    which the last key tile of the sequence before it also covers."""
    lens = [200, 300, 130]
    H = 2
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    T = int(cu[-1])
    if kind == "fp8":
        q, k, v = (_codes(T, H, s, 6.0) for s in (41, 42, 43))
        bad = 0x7F                                     # E4M3 NaN
        v[210, 0, 5] = bad                             # sequence 1, row 10
        v[255, 1, 77] = bad | 0x80                     # sequence 1, row 55 (tile end)
        k[203, 0, 0] = bad                             # a key of sequence 1
        q[220, 1, 9] = bad                             # a query of sequence 1
        v[505, 0, 3] = bad                             # sequence 2, row 5
    else:
        qf, kf, vf, _ = synthetic.small_qkv(44, lens, H=H, scale=1.5)
        v = vf.float() * (1.0 / 15.0)
        v[210, 0, 5] = float("inf")
        v[255, 1, 77] = float("nan")
        v[505, 0, 3] = float("-inf")
        kf = kf.float()
        kf[203, 0, 0] = float("nan")
        q, k, v = qf, kf.to(torch.bfloat16), v.to(torch.bfloat16)
    return lens, H, cu, q, k, v


@pytest.mark.parametrize("rule,orule", RULES)
def test_fp8_nan_in_the_next_sequence_does_not_leak(rule, orule):
    """A NaN code in sequence b+1 within the last, partial key tile of
    sequence b: sequence b must match the oracle (which attends only to its
    own keys), and the sequences holding NaN must be NaN exactly where the
    oracle's output is."""
    lens, H, cu, q8, k8, v8 = _nan_boundary_case("fp8")
    ds = [0.05, 0.04, 1.0 / 60.0]
    out = qar.varlen_fwd(q8.to(DEV), k8.to(DEV), v8.to(DEV), torch.as_tensor(cu, device=DEV),
                         max(lens), torch.tensor(ds, device=DEV), p_rule=rule)
    want = oracle.attention_fp8(q8.numpy(), k8.numpy(), v8.numpy(), cu, ds,
                                return_alternative=True, rule=orule)
    seq0 = np.arange(cu[0], cu[1])
    assert np.isfinite(out[:cu[1]].float().cpu().numpy()).all()
    assert_attention_close(out, tuple(w[seq0] for w in want), rows=seq0,
                           what=f"fp8 NaN next {orule}")
    assert_attention_close(out, want, what=f"fp8 NaN all {orule}")


def test_bf16_inf_and_nan_in_the_next_sequence_do_not_leak():
    lens, H, cu, q, k, v = _nan_boundary_case("bf16")
    out = qar.varlen_fwd_bf16(q.to(DEV), k.to(DEV), v.to(DEV), torch.as_tensor(cu, device=DEV),
                              max(lens))
    want = oracle.attention_bf16(bits(q), bits(k), bits(v), cu)
    seq0 = np.arange(cu[0], cu[1])
    assert np.isfinite(out[:cu[1]].float().cpu().numpy()).all()
    assert_attention_close(out, want[seq0], rows=seq0, what="bf16 Inf/NaN next")
    assert_attention_close(out, want, what="bf16 Inf/NaN all")


def test_bad_cu_seqlens_sets_error_word():
    cu = torch.tensor([0, 100, 50], dtype=torch.int32, device=DEV)   # decreasing
    q8 = torch.zeros(300, 1, 128, dtype=torch.uint8, device=DEV)
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    out = torch.full((300, 1, 128), 7.0, dtype=torch.bfloat16, device=DEV)
    qar.varlen_fwd(q8, q8, q8, cu, 300, torch.ones(3, device=DEV), out=out, error=err)
    assert qar.read_error_word(err) == 6
    assert (out[100:] == 7.0).all()       # the broken sequence wrote nothing
    assert (out[:100] == 0.0).all()       # the valid one attends to zeros
    assert qar.read_error_word(err) == 0


@pytest.mark.parametrize("rule,orule", RULES)
def test_reference_max_stays_and_moves_by_design(rule, orule):
    """Block maxima chosen so the reference max stays within the lag (block 1:
    +1.5 = +2.16 in log2 units), moves past it (block 2: +3.0 over the
    reference = +4.33), stays again (block 3), and sees a lower block (4);
    the other keys score below 0.6.  Exercised for rows of both query tiles."""
    n, H, D = 5 * 128, 1, 128
    cu = np.array([0, n], dtype=np.int32)
    g = torch.Generator().manual_seed(21)
    q = torch.zeros(n, H, D)
    q[:, :, 0] = 1.0
    k = torch.zeros(n, H, D)
    k[:, :, 0] = torch.rand(n, H, generator=g) * 0.6          # background scores
    for blk, x in enumerate((1.0, 2.5, 4.0, 5.5, 3.0)):       # one maximum per block
        k[128 * blk + 17, :, 0] = x
    v = torch.randn(n, H, D, generator=g) * 0.5
    q8, k8, v8 = (t.to(torch.float8_e4m3fn).view(torch.uint8) for t in (q, k, v))
    ds = [1.0, 1.0, 1.0]
    out = qar.varlen_fwd(q8.to(DEV), k8.to(DEV), v8.to(DEV), torch.as_tensor(cu, device=DEV), n,
                         torch.tensor(ds, device=DEV), softmax_scale=1.0, p_rule=rule)
    want = oracle.attention_fp8(q8.numpy(), k8.numpy(), v8.numpy(), cu, ds, scale=1.0,
                                return_alternative=True, rule=orule)
    assert np.isfinite(want[1]).all()                         # no decision at a tie
    assert_attention_close(out, want, what=f"reference max stays and moves {orule}")
