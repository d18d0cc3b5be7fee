"""GPU tests of the static-scale cast fused into the FP8 attention kernel
(``Context.varlen_fwd_static``, C entry point ``fp8attn_varlen_fwd_static``).

The fused call must reproduce, bit for bit, the two-launch path it replaces
(the STATIC cast into E4M3 codes, then the FP8 attention on those codes with
the layer's descales): the cast is the same fl32(x * qs) rounded to nearest
even E4M3 with saturation, only done on shared-memory tiles inside the
attention kernel.  One case is also checked against the oracle directly."""
import numpy as np
import pytest
import torch

import oracle
import synthetic
import quantization_amax_reduce_b200 as qar
from tests.parity import OracleLayer, assert_attention_close, bits, sample_rows

pytestmark = pytest.mark.gpu

DEV = "cuda"
RULES = [pytest.param(qar.P_LINEAR_LOG, id="linear_log"), pytest.param(qar.P_EXP2, id="exp2")]
BOUNDS = (224.0, 198.0, 210.0)


def _bf16(T, H, seed, scale):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(T, H, 128, generator=g) * scale).to(torch.bfloat16).to(DEV)


def _two_launch(ctx, q, k, v, cu_d, S, rule):
    q8, k8, v8 = ctx.quantize_qkv(0, qar.STATIC, q, k, v, cu_d, S)
    return qar.varlen_fwd(q8, k8, v8, cu_d, S, ctx.descale_ptr(0), p_rule=rule)


CASES = [
    ([1], 1), ([5], 2), ([128], 1), ([129], 1), ([256], 2), ([300], 3), ([1000, 17], 2),
    ([64, 0, 200, 0], 2), ([5, 300, 129], 3), ([513, 1, 255], 1),
    # whole waves: both launches of the automatic schedule (whole units, then
    # single-tile CTAs) and the all-split single wave
    ([257, 1, 129], 60), ([1000, 17], 40), ([2000], 16),
]


@pytest.mark.parametrize("rule", RULES)
@pytest.mark.parametrize("lens,H", CASES)
def test_fused_equals_cast_then_attention(lens, H, rule):
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    T, S = int(cu[-1]), int(max(lens))
    q, k, v = (_bf16(T, H, s, 1.5) for s in (11, 12, 13))
    cu_d = torch.as_tensor(cu, device=DEV)
    ctx = qar.Context(1)
    ctx.set_static_scales(0, *BOUNDS)
    want = _two_launch(ctx, q, k, v, cu_d, S, rule)
    got = ctx.varlen_fwd_static(0, q, k, v, cu_d, S, p_rule=rule)
    torch.cuda.synchronize()
    assert torch.equal(got, want), f"{lens} H={H}: max |diff| " \
        f"{(got.float() - want.float()).abs().max().item()}"
    assert ctx.get_error() == 0


@pytest.mark.parametrize("rule", RULES)
def test_fused_reads_an_interleaved_projection(rule):
    """q, k, v as slices of one [T, 3, H, 128] tensor (row stride 3 H 128)."""
    lens, H = [700, 33, 1300], 6
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    T, S = int(cu[-1]), max(lens)
    g = torch.Generator().manual_seed(21)
    qkv = (torch.randn(T, 3, H, 128, generator=g) * 2.0).to(torch.bfloat16).to(DEV)
    q, k, v = qkv[:, 0], qkv[:, 1], qkv[:, 2]
    cu_d = torch.as_tensor(cu, device=DEV)
    ctx = qar.Context(1)
    ctx.set_static_scales(0, 30.0, 25.0, 12.0)
    want = _two_launch(ctx, q, k, v, cu_d, S, rule)
    got = ctx.varlen_fwd_static(0, q, k, v, cu_d, S, p_rule=rule)
    assert torch.equal(got, want)
    # the same through packed copies
    got2 = ctx.varlen_fwd_static(0, q.contiguous(), k.contiguous(), v.contiguous(), cu_d, S,
                                 p_rule=rule)
    assert torch.equal(got2, want)


def test_fused_sets_the_layer_scales_like_the_cast():
    lens, H = [400, 90], 4
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    T = int(cu[-1])
    q, k, v = (_bf16(T, H, s, 1.0) for s in (1, 2, 3))
    cu_d = torch.as_tensor(cu, device=DEV)
    a, b = qar.Context(1), qar.Context(1)
    for c in (a, b):
        c.set_static_scales(0, *BOUNDS)
    a.quantize_qkv(0, qar.STATIC, q, k, v, cu_d, 400)
    b.varlen_fwd_static(0, q, k, v, cu_d, 400)
    qa, da = a.get_scales(0)
    qb, db = b.get_scales(0)
    assert np.array_equal(qa, qb) and np.array_equal(da, db)
    assert da[0] == 0.5 and qa[0] == 2.0


def test_fused_c3_full_size_bit_exact_and_against_the_oracle():
    """S=8192, 16 heads, static 224/198/210: the whole output equals the
    two-launch path; sampled rows match the oracle's attention on the
    oracle's own codes and descales."""
    q, k, v, cu = synthetic.qkv(3, device=DEV)
    cu_d = torch.as_tensor(cu, device=DEV)
    ctx = qar.Context(1)
    ctx.set_static_scales(0, *BOUNDS)
    want = _two_launch(ctx, q, k, v, cu_d, 8192, qar.P_LINEAR_LOG)
    got = ctx.varlen_fwd_static(0, q, k, v, cu_d, 8192)
    assert torch.equal(got, want)
    ol = OracleLayer()
    ol.set_static(BOUNDS)
    codes = ol.static_pass([bits(q), bits(k), bits(v)], cu, 16)
    rows = sample_rows(cu, 64, seed=9)
    ref = oracle.attention_fp8(*codes, cu, [float(x) for x in ol.ds], rows=rows,
                               return_alternative=True, rule=oracle.P_LINEAR_LOG)
    assert_attention_close(got, ref, rows=rows, what="fused static c3")
    assert ctx.get_error() == 0


@pytest.mark.parametrize("rule", RULES)
def test_fused_nan_in_the_next_sequence_does_not_leak(rule):
    """Sequence 0 ends mid-tile; the first rows of sequence 1 hold NaN in V
    (cast to the E4M3 NaN code).  Sequence 0 must not see them."""
    lens, H = [300, 200], 2
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    T = int(cu[-1])
    q, k, v = (_bf16(T, H, s, 1.0) for s in (5, 6, 7))
    v[300:330] = float("nan")
    cu_d = torch.as_tensor(cu, device=DEV)
    ctx = qar.Context(1)
    ctx.set_static_scales(0, *BOUNDS)
    got = ctx.varlen_fwd_static(0, q, k, v, cu_d, 300, p_rule=rule)
    assert torch.isfinite(got[:300]).all()
    want = _two_launch(ctx, q, k, v, cu_d, 300, rule)
    assert torch.equal(got[:300], want[:300])


def test_fused_needs_static_scales_and_packed_rows():
    q = _bf16(10, 2, 1, 1.0)
    cu_d = torch.as_tensor(np.array([0, 10], dtype=np.int32), device=DEV)
    ctx = qar.Context(2)
    with pytest.raises(qar.FP8AttnError):
        ctx.varlen_fwd_static(0, q, q, q, cu_d, 10)       # no static scales yet
    ctx.set_static_scales(1, *BOUNDS)
    with pytest.raises(qar.FP8AttnError):
        ctx.varlen_fwd_static(2, q, q, q, cu_d, 10)       # no such layer
    ctx.varlen_fwd_static(1, q, q, q, cu_d, 10)
    # heads overlapping within a row: refused before any launch
    wide = torch.zeros(10, 2, 256, dtype=torch.bfloat16, device=DEV)
    over = wide.as_strided((10, 2, 128), (256, 64, 1))
    with pytest.raises(qar.FP8AttnError):
        ctx.varlen_fwd_static(1, over, over, over, cu_d, 10)
    assert ctx.get_error() == 0


def test_fused_bad_cu_seqlens_sets_the_context_error():
    """A decreasing cu_seqlens: the broken sequence writes nothing and the
    context's error word reports SEQLENS; the valid one is computed."""
    cu = torch.tensor([0, 100, 50], dtype=torch.int32, device=DEV)
    q = torch.zeros(300, 1, 128, dtype=torch.bfloat16, device=DEV)
    out = torch.full((300, 1, 128), 7.0, dtype=torch.bfloat16, device=DEV)
    ctx = qar.Context(1)
    ctx.set_static_scales(0, *BOUNDS)
    ctx.varlen_fwd_static(0, q, q, q, cu, 300, out=out)
    assert ctx.get_error() == 6
    assert (out[100:] == 7.0).all()
    assert (out[:100] == 0.0).all()
    assert ctx.get_error() == 0
