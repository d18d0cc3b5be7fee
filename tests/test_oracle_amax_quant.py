"""Pins for the oracle's amax and cast over packed, padded and interleaved
sources (CPU only).

vLLM docs, "FP8 ViT encoder attention", notes: quantisation before the
attention call costs quant launches plus an unpadding step -- so the cast
reads only the valid tokens of each sequence and writes them packed.
"""
import numpy as np
import torch

import oracle
import synthetic
from tests.fp_helpers import brute_force_e4m3


def _pad(x, cu, S_max, fill):
    """Scatter packed [T,H,D] into a padded [B,S_max,H,D] filled with `fill`."""
    B = len(cu) - 1
    T, H, D = x.shape
    out = torch.full((B, S_max, H, D), fill, dtype=x.dtype)
    for b in range(B):
        n = cu[b + 1] - cu[b]
        out[b, :n] = x[cu[b]:cu[b + 1]]
    return out


def test_amax_matches_numpy_and_ignores_nan():
    q, k, v, cu = synthetic.small_qkv(1, [5, 17, 3], H=3, D=128, scale=2.0)
    bits = synthetic.bf16_bits(q)
    a, nf = oracle.amax(bits, cu, 3, 128)
    ref = np.abs(q.float().numpy()).max()
    assert a == np.float32(ref) and not nf
    # NaN anywhere is ignored
    qn = q.clone()
    qn[4, 1, 7] = float("nan")
    a2, nf2 = oracle.amax(synthetic.bf16_bits(qn), cu, 3, 128)
    assert a2 == np.float32(np.nanmax(np.abs(qn.float().numpy()))) and not nf2
    # an infinity is reported as non-finite
    qi = q.clone()
    qi[0, 0, 0] = float("-inf")
    a3, nf3 = oracle.amax(synthetic.bf16_bits(qi), cu, 3, 128)
    assert nf3 and np.isinf(a3)


def test_amax_excludes_padding():
    q, _, _, cu = synthetic.small_qkv(2, [7, 2, 11], H=2, D=128)
    S_max = 16
    padded = _pad(q, cu, S_max, 1e30)
    start = np.arange(3, dtype=np.int32) * S_max
    a, nf = oracle.amax(synthetic.bf16_bits(padded), cu, 2, 128, tok_stride=2 * 128,
                        head_stride=128, src_seq_start=start)
    assert a == np.float32(np.abs(q.float().numpy()).max()) and not nf


def _reference_codes(x, qs):
    y = x.float().numpy() * np.float32(qs)      # one fp32 RN multiply
    return brute_force_e4m3(y.astype(np.float64)).reshape(x.shape)


def test_quantize_packed_matches_bruteforce():
    q, _, _, cu = synthetic.small_qkv(3, [9, 4], H=2, D=128, scale=30.0)
    qs = np.float32(448.0) / np.float32(97.0)
    got = oracle.quantize(synthetic.bf16_bits(q), cu, 2, 128, qs)
    np.testing.assert_array_equal(got, _reference_codes(q, qs))


def test_quantize_unpads_padded_source():
    q, _, _, cu = synthetic.small_qkv(4, [3, 8, 1], H=2, D=128)
    S_max = 10
    padded = _pad(q, cu, S_max, 7e4)
    start = np.arange(3, dtype=np.int32) * S_max
    qs = np.float32(2.5)
    got = oracle.quantize(synthetic.bf16_bits(padded), cu, 2, 128, qs, tok_stride=256,
                          head_stride=128, src_seq_start=start)
    np.testing.assert_array_equal(got, _reference_codes(q, qs))


def test_quantize_interleaved_qkv_source():
    # a fused [T, 3, H, D] projection output read through strides
    q, k, v, cu = synthetic.small_qkv(5, [6, 5], H=3, D=128)
    qkv = torch.stack([q, k, v], dim=1).contiguous()        # [T, 3, H, D]
    bits = synthetic.bf16_bits(qkv).reshape(-1)
    T, H, D = q.shape
    for i, t in enumerate((q, k, v)):
        sub = bits[i * H * D:]
        got = oracle.quantize(sub, cu, H, D, 3.0, tok_stride=3 * H * D, head_stride=D)
        np.testing.assert_array_equal(got, _reference_codes(t, 3.0))
        a, _ = oracle.amax(sub, cu, H, D, tok_stride=3 * H * D, head_stride=D)
        assert a == np.float32(np.abs(t.float().numpy()).max())


def test_quantize_saturates_and_keeps_sign():
    x = torch.tensor([[[500.0, -500.0, 0.0, -0.0] + [1.0] * 124]], dtype=torch.bfloat16)
    cu = np.array([0, 1], dtype=np.int32)
    got = oracle.quantize(synthetic.bf16_bits(x), cu, 1, 128, 1.0)
    assert got[0, 0, :4].tolist() == [0x7E, 0xFE, 0x00, 0x80]
