"""The FP8 kernel's polynomial exp2 (f2_exp2_poly in csrc/sm100_ptx.cuh),
emulated step by step in fp32 on the CPU against fp64 2^x.

The kernel evaluates 2^x on the FMA pipe for some of its exponentials: x = j
+ f with j the nearest integer (1.5 * 2^23 added and removed), f = x - j in
[-1/2, 1/2], 2^f from a degree-5 polynomial in Horner form (fused
multiply-adds), and j added into the exponent bits.  Its header states a
maximum relative error of 2.13e-7 on [-126, 8]; the oracle's tie model allows
2^-21 (4.8e-7) for any exp2 the kernel evaluates.  The coefficients are read
from the header, so this pins the polynomial the kernel is compiled with."""
import os
import re

import numpy as np

from tests.conftest import ROOT

HEADER = os.path.join(ROOT, "quantization_amax_reduce_b200", "csrc", "sm100_ptx.cuh")


def _coefficients():
    src = open(HEADER).read()
    body = src[src.index("f2_exp2_poly(uint64_t x)"):]
    body = body[:body.index("\n}\n")]
    lits = re.findall(r"f2_pack\(([-0-9.eE]+)f, \1f\)", body)
    vals = [np.float32(float(v)) for v in lits]
    # the shift constants come first (1.5 * 2^23, -1.5 * 2^23, -1), then the
    # six Horner coefficients from the highest degree down
    assert vals[:3] == [np.float32(12582912.0), np.float32(-12582912.0), np.float32(-1.0)]
    return vals[3:]


def _fma32(a, b, c):
    """fp32 fused multiply-add: a*b is exact in fp64 for fp32 inputs, and the
    sum is rounded once to extended precision before the fp32 rounding
    (double rounding only at exact ties of the second rounding, far below
    the tolerances checked here)."""
    return np.float32(np.longdouble(a) * np.longdouble(b) + np.longdouble(c))


def _emulate(x):
    x = x.astype(np.float32)
    r = (x + np.float32(12582912.0)).astype(np.float32)           # add.rn.f32
    j = (r - np.float32(12582912.0)).astype(np.float32)           # exact
    f = _fma32(j, np.float32(-1.0), x)                             # x - j, exact
    c = _coefficients()
    p = np.full_like(f, c[0])
    for ck in c[1:]:
        p = _fma32(p, f, ck)
    bits = p.view(np.uint32) + (r.view(np.uint32) << np.uint32(23))
    return bits.view(np.float32)


def test_polynomial_exp2_error_bound():
    c = _coefficients()
    assert len(c) == 6
    xs = [np.linspace(-126.0, 8.0, 1 << 21, dtype=np.float32),
          np.linspace(-0.5, 0.5, 1 << 20, dtype=np.float32),
          # around the points where the nearest integer changes
          (np.arange(-126, 8) + 0.5).astype(np.float32)[:, None]
          + np.float32(2.0 ** -20) * np.arange(-64, 65, dtype=np.float32)[None, :]]
    worst = 0.0
    for x in xs:
        x = np.clip(x.ravel(), -126.0, 8.0).astype(np.float32)
        got = _emulate(x).astype(np.float64)
        want = np.exp2(x.astype(np.float64))
        worst = max(worst, float(np.max(np.abs(got - want) / want)))
    print(f"max relative error of the polynomial exp2 on [-126, 8]: {worst:.3e}")
    assert worst <= 2.13e-7 * 1.05
    assert worst <= 2.0 ** -21
