"""Pins for the oracle's fp64 attention (CPU only).

vLLM-Omni docs, "Quantized KV Cache", overview: Q/K/V are quantised
dynamically right before the (full, non-causal) attention operator.  The
pages give no numeric attention outputs, so the oracle is pinned by a
library special case (softmax from scipy with no P quantisation), closed
forms (Q = 0, a single key, hand-worked cases that exercise the block rule
e4m3(32 exp(s - r)) with its lagged reference max r), and invariants.
"""
import math

import numpy as np
import pytest
import scipy.special
import torch

import oracle
import synthetic


def _codes(shape, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(*shape, generator=g) * scale
    return x.to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def _decode_torch(codes):
    return torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()


def _softmax_attention(q, k, v, cu, scale):
    """Library special case: per sequence and head, softmax(q k^T s) v."""
    T, H, D = q.shape
    out = np.empty((T, H, D))
    for b in range(len(cu) - 1):
        s0, s1 = cu[b], cu[b + 1]
        for h in range(H):
            S = q[s0:s1, h] @ k[s0:s1, h].T * scale
            out[s0:s1, h] = scipy.special.softmax(S, axis=-1) @ v[s0:s1, h]
    return out


@pytest.mark.parametrize("lens", [[1, 5, 16], [8], [3, 3]])
def test_unquantized_p_matches_library_softmax(lens):
    H, D = 2, 128
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    T = int(cu[-1])
    q8, k8, v8 = (_codes((T, H, D), s, 2.0) for s in (1, 2, 3))
    ds = (0.031, 0.07, 1.7)
    scale = 1.0 / math.sqrt(D)
    got = oracle.attention_fp8(q8, k8, v8, cu, ds, pquant=False, rule=oracle.P_EXP2)
    want = _softmax_attention(_decode_torch(q8) * ds[0], _decode_torch(k8) * ds[1],
                              _decode_torch(v8) * ds[2], cu, scale)
    np.testing.assert_allclose(got, want, rtol=1e-11, atol=1e-13)


def test_bf16_attention_matches_library_softmax():
    q, k, v, cu = synthetic.small_qkv(9, [4, 13], H=2, D=128)
    got = oracle.attention_bf16(synthetic.bf16_bits(q), synthetic.bf16_bits(k),
                                synthetic.bf16_bits(v), cu)
    f = lambda t: t.to(torch.float64).numpy()
    want = _softmax_attention(f(q), f(k), f(v), cu, 1.0 / math.sqrt(128))
    np.testing.assert_allclose(got, want, rtol=1e-11, atol=1e-13)


def test_zero_query_gives_mean_of_v_exactly_even_with_pquant():
    # every score is 0, so p = 1, 256 p = 256 is an E4M3 value, p~ = 1
    T, H, D = 37, 2, 128
    cu = np.array([0, T], dtype=np.int32)
    q8 = np.zeros((T, H, D), np.uint8)
    k8, v8 = _codes((T, H, D), 4), _codes((T, H, D), 5)
    ds_v = 0.75
    got = oracle.attention_fp8(q8, k8, v8, cu, (0.5, 0.5, ds_v), pquant=True, rule=oracle.P_EXP2)
    mean_v = _decode_torch(v8).mean(axis=0) * ds_v
    for t in range(T):
        np.testing.assert_allclose(got[t], mean_v, rtol=1e-14, atol=1e-15)


def test_single_key_returns_that_value():
    H, D = 3, 128
    cu = np.array([0, 1, 2], dtype=np.int32)        # two sequences of length 1
    q8, k8, v8 = (_codes((2, H, D), s, 3.0) for s in (6, 7, 8))
    got = oracle.attention_fp8(q8, k8, v8, cu, (1.3, 0.2, 0.4), pquant=True, rule=oracle.P_EXP2)
    np.testing.assert_array_equal(got, _decode_torch(v8) * 0.4)


def _two_key_case(s1_code):
    """q = e_0, k0 = 0, k1 = value(s1_code) e_0, v0 = 0, v1 = e_1; unit scales."""
    D = 128
    q8 = np.zeros((2, 1, D), np.uint8)
    k8 = np.zeros((2, 1, D), np.uint8)
    v8 = np.zeros((2, 1, D), np.uint8)
    q8[:, 0, 0] = 0x38            # 1.0
    k8[1, 0, 0] = s1_code
    v8[1, 0, 1] = 0x38            # v1 = e_1
    cu = np.array([0, 2], dtype=np.int32)
    return q8, k8, v8, cu


def test_pquant_rule_normal_range():
    # s = (0, -0.125): r = 0, p1 = e^-0.125 = 0.88250; 32 p1 = 28.24 lies in
    # [16, 32) where E4M3 spacing is 2, nearest 28 -> p~1 = 28/32 = 0.875.
    # l is the unquantised sum 1 + e^-0.125.
    q8, k8, v8, cu = _two_key_case(0xA0)      # 0xA0 = -0.125
    o = oracle.attention_fp8(q8, k8, v8, cu, (1.0, 1.0, 1.0), scale=1.0, pquant=True, rule=oracle.P_EXP2)
    want = 0.875 / (1.0 + math.exp(-0.125))
    assert abs(o[0, 0, 1] - want) < 1e-15
    assert o[0, 0, 0] == 0.0
    # the unquantised and the "l = sum p~" variants differ visibly
    o_none = oracle.attention_fp8(q8, k8, v8, cu, (1, 1, 1), scale=1.0, pquant=False, rule=oracle.P_EXP2)
    assert abs(o_none[0, 0, 1] - math.exp(-0.125) / (1 + math.exp(-0.125))) < 1e-15
    o_lq = oracle.attention_fp8(q8, k8, v8, cu, (1, 1, 1), scale=1.0, pquant=True,
                                l_of_quantized=True, rule=oracle.P_EXP2)
    assert abs(o_lq[0, 0, 1] - 0.875 / 1.875) < 1e-15


def test_pquant_rule_subnormal_range():
    # s = (0, -8): p1 = e^-8 = 3.3546e-4; 32 p1 = 0.010735 is below 2^-6, in
    # the subnormal range with spacing 2^-9: 0.010735 / 2^-9 = 5.496 rounds
    # to 5, so p~1 = 5 * 2^-9 / 32 = 5 * 2^-14.
    q8, k8, v8, cu = _two_key_case(0xD0)      # 0xD0 = -8.0
    o = oracle.attention_fp8(q8, k8, v8, cu, (1.0, 1.0, 1.0), scale=1.0, pquant=True, rule=oracle.P_EXP2)
    want = 5 * 2.0 ** -14 / (1.0 + math.exp(-8.0))
    assert abs(o[0, 0, 1] - want) < 1e-18


def test_rows_sum_to_one_and_columns_stay_in_range():
    H, D = 2, 128
    lens = [40, 7]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    T = int(cu[-1])
    q8, k8, v8 = (_codes((T, H, D), s, 4.0) for s in (10, 11, 12))
    ones = np.full((T, H, D), 0x38, np.uint8)
    o = oracle.attention_fp8(q8, k8, ones, cu, (0.3, 0.3, 1.0), pquant=False, rule=oracle.P_EXP2)
    np.testing.assert_allclose(o, 1.0, rtol=0, atol=1e-14)
    oq = oracle.attention_fp8(q8, k8, ones, cu, (0.3, 0.3, 1.0), pquant=True, rule=oracle.P_EXP2)
    # |p~ - p| <= p / 16 for normal codes; a subnormal code is off by at most
    # half its 2^-9 step, 2^-10 / 32 = 2^-15 per key
    assert np.all(np.abs(oq - 1.0) <= 2.0 ** -4 + 64 * 2.0 ** -15)
    o = oracle.attention_fp8(q8, k8, v8, cu, (0.3, 0.3, 1.0), pquant=False, rule=oracle.P_EXP2)
    vv = _decode_torch(v8)
    for b in range(len(lens)):
        sl = slice(cu[b], cu[b + 1])
        lo, hi = vv[sl].min(axis=0), vv[sl].max(axis=0)
        assert np.all(o[sl] >= lo - 1e-12) and np.all(o[sl] <= hi + 1e-12)


def test_row_subset_equals_full_rows():
    H, D = 2, 128
    cu = np.array([0, 20, 33], dtype=np.int32)
    q8, k8, v8 = (_codes((33, H, D), s, 2.0) for s in (13, 14, 15))
    full = oracle.attention_fp8(q8, k8, v8, cu, (0.1, 0.2, 0.3), rule=oracle.P_EXP2)
    rows = [0, 19, 20, 32, 5]
    sub = oracle.attention_fp8(q8, k8, v8, cu, (0.1, 0.2, 0.3), rows=rows, rule=oracle.P_EXP2)
    np.testing.assert_array_equal(sub, full[rows])


def _block_step_case(s128_code):
    """129 keys, q = e_0: keys 0..127 score 0 (block 0), key 128 scores
    value(s128_code) (block 1); v_128 = e_1, v_0 = e_2; one query row."""
    D, n = 128, 129
    q8 = np.zeros((n, 1, D), np.uint8)
    k8 = np.zeros((n, 1, D), np.uint8)
    v8 = np.zeros((n, 1, D), np.uint8)
    q8[:, 0, 0] = 0x38                # q = e_0
    k8[128, 0, 0] = s128_code
    v8[128, 0, 1] = 0x38              # v_128 = e_1
    v8[0, 0, 2] = 0x38                # v_0 = e_2
    cu = np.array([0, n], dtype=np.int32)
    return q8, k8, v8, cu


def test_reference_max_stays_when_block_max_is_within_the_lag():
    # s_128 = 1 < 3 ln 2 = 2.079 (3 in log2 units): r stays 0 (block 0's
    # max).  Key 128: 32 e^1 = 86.98 lies in [64, 128) with spacing 8 -> 88,
    # carried to the final max 1: p~ = 88/32 e^-1.  Block 0 keys: 32 e^0 = 32
    # exact -> p~ = e^-1.  l = 128 e^-1 + 1 (unquantised).
    q8, k8, v8, cu = _block_step_case(0x38)          # s_128 = 1.0
    o = oracle.attention_fp8(q8, k8, v8, cu, (1.0, 1.0, 1.0), scale=1.0, pquant=True,
                             rows=[5], rule=oracle.P_EXP2)
    l = 128 * math.exp(-1.0) + 1.0
    assert abs(o[0, 0, 1] - 88.0 / 32.0 * math.exp(-1.0) / l) < 1e-15
    assert abs(o[0, 0, 2] - math.exp(-1.0) / l) < 1e-15
    # a reference that followed every new max would give key 128 exactly 1
    assert abs(o[0, 0, 1] - 1.0 / l) > 1e-5


def test_reference_max_moves_past_the_lag():
    # s_128 = 2.5 > 3 ln 2: r moves to 2.5 at block 1, so key 128 gives
    # 32 e^0 = 32 exactly (p~ = 1); block 0 keys were quantised against r = 0
    # (32 exactly) and carry e^-2.5.  l = 128 e^-2.5 + 1.
    q8, k8, v8, cu = _block_step_case(0x42)          # 0x42 = 2.5
    o = oracle.attention_fp8(q8, k8, v8, cu, (1.0, 1.0, 1.0), scale=1.0, pquant=True,
                             rows=[5], rule=oracle.P_EXP2)
    l = 128 * math.exp(-2.5) + 1.0
    assert abs(o[0, 0, 1] - 1.0 / l) < 1e-15
    assert abs(o[0, 0, 2] - math.exp(-2.5) / l) < 1e-15
    # staying at r = 0 would have given e4m3(32 e^2.5) = e4m3(389.8) = 384
    assert abs(o[0, 0, 1] - 384.0 / 32.0 * math.exp(-2.5) / l) > 1e-5


def test_reference_move_at_the_threshold_makes_the_row_unverifiable():
    # s_128 = 3 ln 2 exactly: the move is decided at the tie, either choice is
    # a correct result of the rule, so the row's allowance is infinite
    q8, k8, v8, cu = _block_step_case(0x38)
    o, amb = oracle.attention_fp8(q8, k8, v8, cu, (1.0, 3.0 * math.log(2.0), 1.0), scale=1.0,
                                  pquant=True, rows=[5], return_ambiguity=True, rule=oracle.P_EXP2)
    assert np.isinf(amb).all()
    o, amb = oracle.attention_fp8(q8, k8, v8, cu, (1.0, 2.5, 1.0), scale=1.0,
                                  pquant=True, rows=[5], return_ambiguity=True, rule=oracle.P_EXP2)
    assert np.isfinite(amb).all()


def test_pquant_block_is_128_keys():
    # keys 0..63 score 0, key 64 scores 1: all in block 0 (128 keys), so
    # keys 0..63 are quantised against the block max 1, giving
    # e4m3(32 e^-1)/32 = e4m3(11.77)/32 = 12/32 = 0.375 (with 64-key blocks
    # the reference would be 0, key 64 would stay within the lag, and keys
    # 0..63 would carry e^-1 exactly).
    D, n = 128, 65
    q8 = np.zeros((n, 1, D), np.uint8)
    k8 = np.zeros((n, 1, D), np.uint8)
    v8 = np.zeros((n, 1, D), np.uint8)
    q8[:, 0, 0] = 0x38
    k8[64, 0, 0] = 0x38               # s_64 = 1
    v8[0, 0, 2] = 0x38                # v_0 = e_2
    cu = np.array([0, n], dtype=np.int32)
    o = oracle.attention_fp8(q8, k8, v8, cu, (1.0, 1.0, 1.0), scale=1.0, pquant=True,
                             rows=[0], rule=oracle.P_EXP2)
    l = 64 * math.exp(-1.0) + 1.0
    assert abs(o[0, 0, 2] - 0.375 / l) < 1e-15


def test_pquant_block_rule_second_block_lower_max():
    # block 1's scores are all below block 0's max: the reference stays 0, so
    # p~ = e4m3(32 e^s)/32 for s = -0.125 there: 28/32
    D, n = 128, 130
    q8 = np.zeros((n, 1, D), np.uint8)
    k8 = np.zeros((n, 1, D), np.uint8)
    v8 = np.zeros((n, 1, D), np.uint8)
    q8[:, 0, 0] = 0x38
    k8[128:, 0, 0] = 0xA0             # s = -0.125 for keys 128, 129
    v8[129, 0, 3] = 0x38
    cu = np.array([0, n], dtype=np.int32)
    o = oracle.attention_fp8(q8, k8, v8, cu, (1.0, 1.0, 1.0), scale=1.0, pquant=True,
                             rows=[0], rule=oracle.P_EXP2)
    l = 128 + 2 * math.exp(-0.125)
    assert abs(o[0, 0, 3] - 0.875 / l) < 1e-15


def test_ambiguity_reported_only_at_rounding_ties():
    # s1 = ln(29/32): y1 = 32 e^{s1} = 29 is the tie between the E4M3 values
    # 28 and 30, so both codes are correct results of the rule and the oracle
    # reports the one-step change (2/32) * |v1| / l.
    q8, k8, v8, cu = _two_key_case(0x38)          # k1 = 1.0 * e_0
    ds_k = math.log(29.0 / 32.0)
    o, amb = oracle.attention_fp8(q8, k8, v8, cu, (1.0, ds_k, 1.0), scale=1.0, pquant=True,
                                  return_ambiguity=True, rule=oracle.P_EXP2)
    l = 1.0 + 29.0 / 32.0
    assert abs(amb[0, 0, 1] - (2.0 / 32.0) / l) < 1e-12
    assert amb[0, 0, 0] == 0.0                    # v1 has no component there
    # y1 = 28.24 (s1 = -0.125) is far from any tie: no allowance
    q8, k8, v8, cu = _two_key_case(0xA0)
    o, amb = oracle.attention_fp8(q8, k8, v8, cu, (1.0, 1.0, 1.0), scale=1.0, pquant=True,
                                  return_ambiguity=True, rule=oracle.P_EXP2)
    assert (amb == 0.0).all()


# --------------------------------------------------------------------------
# The tie model: which codes an implementation may decide either way
# --------------------------------------------------------------------------

def _two_key_case_with_cancelling_channels(s1_code, big):
    """_two_key_case, plus (when `big`) two more channels whose products
    +448 and -448 cancel: the score is unchanged but sum |q_d k_d| (the
    scale of the tensor cores' accumulation error) is ~900x larger."""
    q8, k8, v8, cu = _two_key_case(s1_code)
    if big:
        q8[:, 0, 1] = 0x38
        q8[:, 0, 2] = 0x38
        k8[1, 0, 1] = 0x7E            # +448
        k8[1, 0, 2] = 0xFE            # -448
    return q8, k8, v8, cu


def test_exp2_tie_window_grows_with_the_accumulation_scale():
    # y1 = 32 exp(s1) = 29 (1 + 3e-5): 3e-5 above the tie between the E4M3
    # values 28 and 30.  With the score's products all small the
    # implementation's error is ~3e-6 relative and the code is decided; with
    # two cancelling 448 x 1 products it may be off by ~3e-4, so either code
    # is a correct result and an allowance is reported.
    ds_k = math.log(29.0 * (1.0 + 3e-5) / 32.0)
    for big, want_amb in ((False, False), (True, True)):
        q8, k8, v8, cu = _two_key_case_with_cancelling_channels(0x38, big)
        o, amb = oracle.attention_fp8(q8, k8, v8, cu, (1.0, ds_k, 1.0), scale=1.0,
                                      return_ambiguity=True, rule=oracle.P_EXP2)
        assert (amb[0, 0, 1] > 0) == want_amb, (big, amb[0, 0, 1])
        assert abs(o[0, 0, 1] - (30.0 / 32.0) / (1.0 + 29.0 * (1 + 3e-5) / 32.0)) < 1e-12


def test_linear_log_tie_window_grows_with_the_accumulation_scale():
    # 8 t1 + 56 = 94.502: 0.002 code units above the half-integer between
    # codes 94 and 95.  Small products: decided; cancelling 448 x 1 products:
    # within the implementation's error, so an allowance is reported.
    t1 = (94.502 - 56.0) / 8.0
    ds_k = (t1 - 5.0) / math.log2(math.e)          # s1 = ds_k, r = 0
    for big, want_amb in ((False, False), (True, True)):
        q8, k8, v8, cu = _two_key_case_with_cancelling_channels(0x38, big)
        o, amb = oracle.attention_fp8(q8, k8, v8, cu, (1.0, ds_k, 1.0), scale=1.0,
                                      return_ambiguity=True, rule=oracle.P_LINEAR_LOG)
        assert (amb[0, 0, 1] > 0) == want_amb, (big, amb[0, 0, 1])


# --------------------------------------------------------------------------
# The linear-log P rule: code = RNE(8 t + 56) clamped to [0, 128]
# --------------------------------------------------------------------------

def test_linear_log_code_interpolates_between_powers_of_two():
    # t1 = 4.5 exactly (s1 = -ln(2)/2): 8 t + 56 = 92 = 0x5C, exponent field
    # 11, mantissa 4: (1 + 4/8) 2^4 = 24, so p~1 = 24/32 = 0.75 (linear between
    # 2^4 and 2^5) where the exp2 rule gives e4m3(22.63) = 22 -> 0.6875.
    # Key 0 (score 0, the block max): 8 * 5 + 56 = 96 = 0x60 = 32 -> 1.
    # l is the sum of the quantised values, 1 + 0.75.
    q8, k8, v8, cu = _two_key_case(0x38)
    ds_k = -0.5 * math.log(2.0)
    o = oracle.attention_fp8(q8, k8, v8, cu, (1.0, ds_k, 1.0), scale=1.0,
                             rule=oracle.P_LINEAR_LOG)
    assert abs(o[0, 0, 1] - 0.75 / 1.75) < 1e-15
    e = oracle.attention_fp8(q8, k8, v8, cu, (1.0, ds_k, 1.0), scale=1.0, rule=oracle.P_EXP2)
    assert abs(e[0, 0, 1] - 0.6875 / (1.0 + math.sqrt(0.5))) < 1e-15


def test_linear_log_code_rounds_the_fraction_to_eighths():
    # s1 = -0.125: t1 = 5 - 0.18034 = 4.81966, 8 t + 56 = 94.557 -> 95 = 0x5F:
    # exponent 11, mantissa 7: (1 + 7/8) 16 = 30 -> p~1 = 30/32.
    q8, k8, v8, cu = _two_key_case(0xA0)      # k1 = -0.125 e_0
    o = oracle.attention_fp8(q8, k8, v8, cu, (1.0, 1.0, 1.0), scale=1.0,
                             rule=oracle.P_LINEAR_LOG)
    assert abs(o[0, 0, 1] - (30.0 / 32.0) / (1.0 + 30.0 / 32.0)) < 1e-15


def test_linear_log_subnormal_codes_and_the_clamp():
    # s1 = -8: t1 = 5 - 11.5416 = -6.5416, 8 t + 56 = 3.667 -> code 4, an
    # E4M3 subnormal: 4 * 2^-9 = 2^-7, so p~1 = 2^-7 / 32 = 2^-12.
    q8, k8, v8, cu = _two_key_case(0xD0)      # k1 = -8 e_0
    o = oracle.attention_fp8(q8, k8, v8, cu, (1.0, 1.0, 1.0), scale=1.0,
                             rule=oracle.P_LINEAR_LOG)
    assert abs(o[0, 0, 1] - 2.0 ** -12 / (1.0 + 2.0 ** -12)) < 1e-18
    # s1 = -20: 8 t + 56 < 0 -> code 0, the key drops out entirely
    q8, k8, v8, cu = _two_key_case(0xDA)      # k1 = -20 e_0
    o = oracle.attention_fp8(q8, k8, v8, cu, (1.0, 1.0, 1.0), scale=1.0,
                             rule=oracle.P_LINEAR_LOG)
    assert o[0, 0, 1] == 0.0


def test_linear_log_nan_score_gets_code_zero():
    # a NaN key code makes that key's score NaN: its P code is 0, so the
    # output is the other key's value exactly (v0 = e_2 here)
    q8, k8, v8, cu = _two_key_case(0x7F)      # k1 = NaN
    v8[0, 0, 2] = 0x38
    o = oracle.attention_fp8(q8, k8, v8, cu, (1.0, 1.0, 1.0), scale=1.0,
                             rule=oracle.P_LINEAR_LOG)
    assert o[0, 0, 2] == 1.0 and o[0, 0, 1] == 0.0


def test_linear_log_rows_average_exactly():
    # l is the sum of the quantised P, so with v = 1 every output is 1 (up
    # to fp64 rounding), with the reference moving or not
    H, D = 2, 128
    lens = [300, 7]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    T = int(cu[-1])
    g = torch.Generator().manual_seed(17)
    ramp = torch.linspace(0.2, 3.0, T).view(T, 1, 1)
    q8 = (torch.randn(T, H, D, generator=g) * 4).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    k8 = (torch.randn(T, H, D, generator=g) * 4 * ramp).to(torch.float8_e4m3fn).view(
        torch.uint8).numpy()
    ones = np.full((T, H, D), 0x38, np.uint8)
    o = oracle.attention_fp8(q8, k8, ones, cu, (0.25, 0.25, 1.0), rule=oracle.P_LINEAR_LOG)
    np.testing.assert_allclose(o, 1.0, rtol=0, atol=1e-13)


def test_move_at_the_threshold_gives_two_results_not_an_exclusion():
    # block 1's max lies 1e-12 above the move threshold (3 ln 2 over r = 0 in
    # natural units), well inside an implementation's error: with
    # return_alternative the row comes back evaluated both ways (moved and
    # not moved), with finite allowances, instead of being given up.  A
    # second key of block 1 scores 1.0, so the two outcomes quantise it
    # against references 3 ln 2 + 1e-12 apart.
    D, n = 128, 130
    q8 = np.zeros((n, 1, D), np.uint8)
    k8 = np.zeros((n, 1, D), np.uint8)
    v8 = np.zeros((n, 1, D), np.uint8)
    q8[:, 0, 0] = 0x38
    k8[128, 0, 0] = 0x38                  # s = ds_k (the threshold score)
    v8[128, 0, 1] = 0x38
    v8[129, 0, 2] = 0x38
    v8[0, 0, 3] = 0x38
    cu = np.array([0, n], dtype=np.int32)
    ds_k = 3.0 * math.log(2.0) + 1e-12
    k8[129, 0, 0] = 0x38
    for rule in (oracle.P_EXP2, oracle.P_LINEAR_LOG):
        o, amb, alt, alt_amb = oracle.attention_fp8(
            q8, k8, v8, cu, (1.0, ds_k, 1.0), scale=1.0, rows=[0], rule=rule,
            return_alternative=True)
        assert np.isfinite(amb).all() and np.isfinite(alt).all() and np.isfinite(alt_amb).all()
        np.testing.assert_allclose(alt, o, rtol=0.2, atol=1e-6)
        # without the alternative the row is reported as unverifiable
        o2, amb2 = oracle.attention_fp8(q8, k8, v8, cu, (1.0, ds_k, 1.0), scale=1.0, rows=[0],
                                        rule=rule, return_ambiguity=True)
        assert np.isinf(amb2).all()
        np.testing.assert_array_equal(o2, o)
    # a row whose moves are decided away from the threshold has no alternative
    o, amb, alt, alt_amb = oracle.attention_fp8(q8, k8, v8, cu, (1.0, 1.0, 1.0), scale=1.0,
                                                rows=[0], return_alternative=True)
    assert np.isnan(alt).all() and np.isfinite(amb).all()
