"""Pins for the oracle's E4M3 codec (CPU only).

The pages name the format (Ascend quantisation chapter: FP8 E4M3 / E5M2);
its layout and the round-to-nearest-even, saturating rule come from the OCP
8-bit floating point specification.  The oracle is checked against values
written out from that definition, against torch's float8_e4m3fn (a library
routine) and against an exhaustive nearest-value search.
"""
import numpy as np
import pytest
import torch

import oracle
from tests.fp_helpers import brute_force_e4m3, e4m3_positive_values

# (code, value) pairs written out from the format definition
KNOWN = [
    (0x00, 0.0), (0x01, 2.0 ** -9), (0x02, 2.0 ** -8), (0x07, 7 * 2.0 ** -9),
    (0x08, 2.0 ** -6), (0x09, 1.125 * 2.0 ** -6), (0x30, 0.5), (0x38, 1.0),
    (0x39, 1.125), (0x3F, 1.875), (0x40, 2.0), (0x70, 128.0), (0x77, 240.0), (0x78, 256.0),
    (0x7E, 448.0), (0x80, -0.0), (0xB8, -1.0), (0xFE, -448.0), (0x81, -(2.0 ** -9)),
]


def test_known_values():
    codes = np.array([c for c, _ in KNOWN], dtype=np.uint8)
    vals = oracle.e4m3_value(codes)
    for (c, v), got in zip(KNOWN, vals):
        assert got == v, hex(c)
        assert np.signbit(got) == np.signbit(v), hex(c)


def test_nan_codes():
    v = oracle.e4m3_value(np.array([0x7F, 0xFF], dtype=np.uint8))
    assert np.isnan(v).all()
    # no infinities anywhere in the table
    allv = oracle.e4m3_value(np.arange(256, dtype=np.uint8))
    assert not np.isinf(allv).any()
    assert np.isnan(allv).sum() == 2


def test_table_matches_definition_and_torch():
    allv = oracle.e4m3_value(np.arange(256, dtype=np.uint8))
    pos = e4m3_positive_values()
    np.testing.assert_array_equal(allv[:0x7F], pos)
    np.testing.assert_array_equal(allv[0x80:0xFF], -pos)
    # library routine: torch's float8_e4m3fn decode of every code
    t = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn)
    tv = t.to(torch.float64).numpy()
    same = (tv == allv) | (np.isnan(tv) & np.isnan(allv))
    assert same.all()


def test_positive_codes_monotone():
    allv = oracle.e4m3_value(np.arange(0x7F, dtype=np.uint8))
    assert (np.diff(allv) > 0).all()
    assert allv.max() == 448.0


def _bf16_all_values():
    bits = np.arange(1 << 16, dtype=np.uint32) << 16
    return bits.view(np.float32)


@pytest.mark.parametrize("qs", [1.0, 2.0, 448.0 / 210.0, 448.0 / 3.7, 0.03125, 37.5])
def test_encoder_vs_bruteforce_all_bf16_times_scale(qs):
    x = _bf16_all_values()
    with np.errstate(over="ignore", invalid="ignore"):
        y = x * np.float32(qs)          # one fp32 RN multiply
    got = oracle.e4m3_encode(y)
    want = brute_force_e4m3(y.astype(np.float64))
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, [(float(y[i]), hex(got[i]), hex(want[i])) for i in bad[:5]]


def test_encoder_midpoints_and_neighbours():
    pos = e4m3_positive_values()
    mids = (pos[:-1] + pos[1:]) / 2.0           # exact in fp32 (few bits)
    mids = mids.astype(np.float32)
    assert (mids.astype(np.float64) == (pos[:-1] + pos[1:]) / 2.0).all()
    up = np.nextafter(mids, np.float32(np.inf))
    dn = np.nextafter(mids, np.float32(0))
    ys = np.concatenate([mids, up, dn, -mids, -up, -dn, pos.astype(np.float32)])
    got = oracle.e4m3_encode(ys)
    want = brute_force_e4m3(ys.astype(np.float64))
    np.testing.assert_array_equal(got, want)
    # ties go to the even mantissa: every exact midpoint encodes to an even code
    assert (oracle.e4m3_encode(mids) % 2 == 0).all()


def test_encoder_vs_torch_cast_in_range():
    rng = np.random.Generator(np.random.PCG64(7))
    y = (rng.standard_normal(200000) * rng.choice([1e-3, 1e-1, 1, 10, 100], 200000)).astype(np.float32)
    y = y[np.abs(y) < 448.0]
    got = oracle.e4m3_encode(y)
    t = torch.from_numpy(y).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(got, t)


def test_special_values():
    f = np.float32
    cases = [
        (f(np.nan), 0x7F), (-f(np.nan), 0x7F), (f(np.inf), 0x7E), (-f(np.inf), 0xFE),
        (f(448.0), 0x7E), (f(463.99), 0x7E), (f(464.0), 0x7E), (f(1e30), 0x7E),
        (f(-500.0), 0xFE), (f(0.0), 0x00), (f(-0.0), 0x80), (f(-1e-10), 0x80),
        (f(2.0 ** -10), 0x00),            # tie between 0 and 2^-9 -> even (0)
        (f(3 * 2.0 ** -10), 0x02),        # tie between 2^-9 and 2^-8 -> even (2)
        (f(2.0 ** -10 * 1.0000001), 0x01),
        (f(1.0625), 0x38),                # tie 1.0 / 1.125 -> even (1.0)
        (f(1.1875), 0x3A),                # tie 1.125 / 1.25 -> even (1.25)
        (f(240.0 + 8.0), 0x78),           # tie 240 / 256 -> even (256)
    ]
    ys = np.array([c[0] for c in cases], dtype=np.float32)
    got = oracle.e4m3_encode(ys)
    for (y, want), g in zip(cases, got):
        assert g == want, (y, hex(g), hex(want))
