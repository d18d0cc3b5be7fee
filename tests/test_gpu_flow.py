"""Full-size workflows on the GPU: DiT-shaped dynamic attention (S=32760,
40 heads) and the multi-layer calibrate-then-serve flow (24 layers, 16
dynamic passes, export x1.5, static serve, layers 0-2 in bf16).

vLLM docs, "FP8 ViT encoder attention", usage section: calibrate by running
dynamic scaling for 16 passes, save the learned scales multiplied by the
save margin (default 1.5), then serve with the static scales.  vLLM-Omni
docs, "Quantized KV Cache", parameters table: skip-layer selectors."""
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


@pytest.mark.parametrize("rule,orule", [(qar.P_LINEAR_LOG, oracle.P_LINEAR_LOG),
                                        (qar.P_EXP2, oracle.P_EXP2)], ids=["linear_log", "exp2"])
def test_c4_dit_dynamic_full_size(rule, orule):
    q, k, v, cu = synthetic.qkv(4, device=DEV)
    ctx = qar.Context(1)
    cu_d = torch.as_tensor(cu, device=DEV)
    q8, k8, v8 = ctx.quantize_qkv(0, qar.DYNAMIC, q, k, v, cu_d, 32760)
    out = qar.varlen_fwd(q8, k8, v8, cu_d, 32760, ctx.descale_ptr(0), p_rule=rule)
    ol = OracleLayer()
    codes = ol.dynamic_pass([bits(q), bits(k), bits(v)], cu, 40)
    for g, w, n in zip((q8, k8, v8), codes, "qkv"):
        assert_codes_equal(g, w, n)
    assert_scales_equal(ctx, 0, ol)
    ds = [float(x) for x in ol.ds]
    # every head on a few rows ...
    rows = sample_rows(cu, 24, seed=4)
    want = oracle.attention_fp8(*codes, cu, ds, rows=rows, return_alternative=True, rule=orule)
    assert_attention_close(out, want, rows=rows, what=f"c4 all heads {orule}")
    # ... and 1024 rows of the first and the last head, with the error
    # against unquantised fp64 attention on the bf16 inputs
    heads = [0, 39]
    rows = sample_rows(cu, 1024, seed=40)
    sub = [np.ascontiguousarray(c[:, heads]) for c in codes]
    want = oracle.attention_fp8(*sub, cu, ds, rows=rows, return_alternative=True, rule=orule)
    ref = oracle.attention_bf16(*(np.ascontiguousarray(bits(x)[:, heads]) for x in (q, k, v)), cu,
                                rows=rows)
    assert_attention_close(out[:, heads], want, rows=rows, what=f"c4 1024 rows x 2 heads {orule}",
                           unquantized=ref)
    assert ctx.get_error() == 0


@pytest.mark.slow
def test_c5_calibrate_then_serve():
    w = synthetic.WORKLOADS[5]
    L = w.layers
    skip = qar.parse_selector(w.skip_layers, L)
    assert skip == oracle.parse_selector(w.skip_layers, L) == {0, 1, 2}
    ctx = qar.Context(L)
    ols = [OracleLayer() for _ in range(L)]
    mask = np.zeros(L, dtype=np.uint8)
    mask[list(skip)] = 1
    check_layers = {3, 12, L - 1}
    cus = [w.cu_seqlens(l) for l in range(L)]
    # --- calibrate: 16 dynamic passes over fresh draws
    for p in range(w.passes):
        for l in range(L):
            mode = ctx.select_mode(l, mask)
            assert mode == oracle.layer_mode(l, skip, False)
            if mode == qar.SKIP:
                continue
            cu = cus[l]
            cu_d = torch.as_tensor(cu, device=DEV)
            max_len = int(np.diff(cu).max())
            q, k, v, _ = synthetic.qkv(5, l, p, device=DEV)
            q8, k8, v8 = ctx.quantize_qkv(l, qar.DYNAMIC, q, k, v, cu_d, max_len)
            hq, hk, hv = bits(q), bits(k), bits(v)
            if l in check_layers and p in (0, w.passes - 1):
                want = ols[l].dynamic_pass([hq, hk, hv], cu, w.H)
                for g, ww, n in zip((q8, k8, v8), want, "qkv"):
                    assert_codes_equal(g, ww, f"layer {l} pass {p} {n}")
            else:
                for t, x in enumerate((hq, hk, hv)):
                    a, nf = oracle.amax(x, cu, w.H, 128)
                    ols[l].qs[t], ols[l].ds[t] = ols[l].rings[t].dynamic_step(a, nf)
            assert_scales_equal(ctx, l, ols[l])
            assert_ring_equal(ctx, l, ols[l])
    assert ctx.get_error() == 0
    # --- export x1.5 and switch to static scales
    exported = ctx.export_static_scales(qar.DEFAULT_MARGIN)
    for l in range(L):
        if l in skip:
            assert (exported[l] == 0).all()
            continue
        for t in range(3):
            assert exported[l, t] == ols[l].rings[t].export_value(1.5)
        ctx.set_static_scales(l, *exported[l].tolist())
        ols[l].set_static(exported[l])
    # --- serve pass
    serve = w.passes
    for l in sorted(check_layers | {0}):
        cu = cus[l]
        cu_d = torch.as_tensor(cu, device=DEV)
        max_len = int(np.diff(cu).max())
        q, k, v, _ = synthetic.qkv(5, l, serve, device=DEV)
        # 1024 rows per sequence of two heads on the first FP8 layer served,
        # 64 rows of every head on the others
        many = l == min(check_layers)
        rows = sample_rows(cu, 1024 if many else 64, seed=l)
        heads = [0, w.H - 1] if many else list(range(w.H))
        mode = ctx.select_mode(l, mask)
        if mode == qar.SKIP:
            out = qar.varlen_fwd_bf16(q, k, v, cu_d, max_len)
            want = oracle.attention_bf16(bits(q), bits(k), bits(v), cu, rows=rows)
            assert_attention_close(out, want, rows=rows, what=f"c5 serve bf16 layer {l}")
            continue
        assert mode == qar.STATIC
        q8, k8, v8 = ctx.quantize_qkv(l, qar.STATIC, q, k, v, cu_d, max_len)
        codes = ols[l].static_pass([bits(q), bits(k), bits(v)], cu, w.H)
        for g, ww, n in zip((q8, k8, v8), codes, "qkv"):
            assert_codes_equal(g, ww, f"serve layer {l} {n}")
        assert_scales_equal(ctx, l, ols[l])
        out = qar.varlen_fwd(q8, k8, v8, cu_d, max_len, ctx.descale_ptr(l))
        sub = [np.ascontiguousarray(c[:, heads]) for c in codes]
        want = oracle.attention_fp8(*sub, cu, [float(x) for x in ols[l].ds], rows=rows,
                                    return_alternative=True)
        ref = oracle.attention_bf16(*(np.ascontiguousarray(bits(x)[:, heads]) for x in (q, k, v)),
                                    cu, rows=rows)
        assert_attention_close(out[:, heads], want, rows=rows,
                               what=f"c5 serve fp8 layer {l} ({len(heads)} heads)",
                               unquantized=ref)
