"""The tensor cores' fp32 accumulation of an E4M3 score, checked against
exact scores.

The oracle's tie model (which P codes and which reference moves an
implementation may decide either way) assumes that a score carries at most
16 u sum_d |q_d k_d| of accumulation error (u = 2^-24).  This test computes
S = Q K^T through the attention kernel's own MMA sequence
(fp8attn_selftest_qk_scores) on random and adversarial E4M3 tiles and checks
that bound against the exact dot products (fp64, exact for E4M3 products)."""
import numpy as np
import pytest
import torch

import oracle
import quantization_amax_reduce_b200 as qar

pytestmark = pytest.mark.gpu

DEV = "cuda"
U = 2.0 ** -24
BOUND = 16.0      # OR_ACC_ROUNDINGS in the oracle


def _finite_codes(rng, shape):
    c = rng.integers(0, 256, size=shape, dtype=np.uint8)
    c[(c & 0x7F) == 0x7F] ^= 1          # no NaN codes
    return c


def _tiles(seed):
    """Six kinds of 128 x 128 tile pairs, 4 of each."""
    rng = np.random.default_rng(seed)
    # values are clipped to the E4M3 range first (torch maps larger ones to NaN)
    enc = lambda x: torch.from_numpy(np.clip(x, -448.0, 448.0).astype(np.float32)).to(
        torch.float8_e4m3fn).view(torch.uint8).numpy()
    qs, ks = [], []
    for kind in range(6):
        for _ in range(4):
            if kind == 0:      # every finite code, uniformly
                q, k = _finite_codes(rng, (128, 128)), _finite_codes(rng, (128, 128))
            elif kind == 1:    # N(0, 16)
                q, k = enc(4 * rng.standard_normal((128, 128))), enc(4 * rng.standard_normal((128, 128)))
            elif kind == 2:    # log-normal magnitudes (wide dynamic range)
                q = enc(rng.standard_normal((128, 128)) * np.exp(2 * rng.standard_normal((128, 128))))
                k = enc(rng.standard_normal((128, 128)) * np.exp(2 * rng.standard_normal((128, 128))))
            elif kind == 3:    # one 448 per 32-channel group, small values elsewhere
                q = enc(0.02 * rng.standard_normal((128, 128)))
                k = enc(0.02 * rng.standard_normal((128, 128)))
                q[:, ::32] = 0x7E
                k[:, ::32] = 0x7E
            elif kind == 4:    # exact cancellation of two large products
                q = enc(0.05 * rng.standard_normal((128, 128)))
                k = enc(0.05 * rng.standard_normal((128, 128)))
                q[:, :2] = 0x7E
                k[:, 0], k[:, 1] = 0x7E, 0xFE
            else:              # a large shared low-rank component (DiT-like)
                q = enc(3 * rng.standard_normal((128, 128)) + 6 * (np.arange(128) < 8))
                k = enc(3 * rng.standard_normal((128, 128)) + 6 * (np.arange(128) < 8))
            qs.append(q)
            ks.append(k)
    return np.concatenate(qs), np.concatenate(ks)


def test_score_accumulation_error_is_within_the_oracle_bound():
    q8, k8 = _tiles(5)
    S = qar.selftest_qk_scores(torch.from_numpy(q8).to(DEV), torch.from_numpy(k8).to(DEV))
    S = S.cpu().numpy().astype(np.float64)
    qv = oracle.e4m3_value(q8).reshape(-1, 128, 128)
    kv = oracle.e4m3_value(k8).reshape(-1, 128, 128)
    exact = np.einsum("tid,tjd->tij", qv, kv)        # exact: E4M3 products fit fp64
    mag = np.einsum("tid,tjd->tij", np.abs(qv), np.abs(kv))
    err = np.abs(S - exact)
    ratio = np.where(mag > 0, err / (U * np.maximum(mag, 1e-300)), 0.0)
    worst = float(ratio.max())
    print(f"max |S - exact| / (u sum|qk|) = {worst:.3f} (bound {BOUND})")
    assert np.isfinite(S).all()
    assert worst <= BOUND, worst
    # the bound is not vacuous: the products are not all summed exactly
    assert (err > 0).any()
