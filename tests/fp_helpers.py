"""Independent exact-arithmetic helpers for pinning the oracle.

Nothing here is shared with the oracle or the CUDA library: rational
rounding to fp32 and a brute-force nearest-E4M3 search built from the
format's definition (the OCP 8-bit floating point spec, E4M3 "FN").
"""
from fractions import Fraction

import numpy as np


def fl32_of_rational(x: Fraction) -> np.float32:
    """Correctly rounded (nearest, ties to even) fp32 of a positive rational."""
    assert x > 0
    e = x.numerator.bit_length() - x.denominator.bit_length()
    # normalise to m in [2^23, 2^24)
    while Fraction(2) ** e > x:
        e -= 1
    while Fraction(2) ** (e + 1) <= x:
        e += 1
    scaled = x / (Fraction(2) ** (e - 23))
    n = scaled.numerator // scaled.denominator
    rem = scaled - n
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and n % 2 == 1):
        n += 1
    return np.float32(float(Fraction(n) * Fraction(2) ** (e - 23)))


def e4m3_positive_values() -> np.ndarray:
    """Values of codes 0x00..0x7E straight from the format definition."""
    vals = []
    for code in range(0x7F):
        e, m = code >> 3, code & 7
        if e == 0:
            vals.append(m / 8.0 * 2.0 ** -6)
        else:
            vals.append((1.0 + m / 8.0) * 2.0 ** (e - 7))
    return np.array(vals, dtype=np.float64)


def brute_force_e4m3(y: np.ndarray) -> np.ndarray:
    """Nearest finite E4M3 value by exhaustive search; equal distances go to
    the code with an even mantissa; NaN -> 0x7F; sign kept (incl. -0)."""
    y = np.asarray(y, dtype=np.float64).reshape(-1)
    table = e4m3_positive_values()
    codes = np.empty(y.size, dtype=np.uint8)
    nan = np.isnan(y)
    # every magnitude >= 448 has 448 as its nearest finite value; clamping
    # keeps the fp64 distances below exact for huge inputs and infinities
    a = np.minimum(np.abs(np.where(nan, 0.0, y)), 1024.0)
    out = np.empty(y.size, dtype=np.int64)
    step = 1 << 16
    for s in range(0, y.size, step):
        blk = a[s:s + step]
        dist = np.abs(blk[:, None] - table[None, :])
        best = dist.min(axis=1, keepdims=True)
        cand = dist == best
        # among equal-distance candidates prefer even codes (even mantissa)
        even = cand & ((np.arange(0x7F) % 2) == 0)[None, :]
        pick_even = even.any(axis=1)
        first_even = np.argmax(even, axis=1)
        first_any = np.argmax(cand, axis=1)
        out[s:s + step] = np.where(pick_even, first_even, first_any)
    codes[:] = out.astype(np.uint8)
    codes |= np.where(np.signbit(y) & ~nan, 0x80, 0).astype(np.uint8)
    codes[nan] = 0x7F
    return codes
