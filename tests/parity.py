"""Shared helpers for the GPU parity tests: run the CUDA path through the
C-ABI binding, run the oracle on the same seeded inputs, compare."""
from __future__ import annotations

import math
from typing import Optional, Sequence

import numpy as np
import torch

import oracle
import synthetic

# Attention tolerance against the oracle (fp64 with the same P rule):
# max err <= 1e-2 and mean err <= 1e-3, with err = |got - ref| / max(1, |ref|).
# For outputs of magnitude <= 1 this is the absolute error; above 1 it is
# relative, because a bf16 output cannot hold a value of magnitude >= 4 to
# within 1e-2 (half a bf16 ulp there is 1/64).
MAX_ABS_TOL = 1e-2
MEAN_ABS_TOL = 1e-3


class OracleLayer:
    """Oracle twin of one layer's device state: three rings + static bounds."""

    def __init__(self):
        self.rings = [oracle.Ring() for _ in range(3)]
        self.static = None
        self.qs = [np.float32(1.0)] * 3
        self.ds = [np.float32(1.0)] * 3

    def dynamic_pass(self, tensors_u16, cu, H, D=128, **src):
        codes = []
        for t, x in enumerate(tensors_u16):
            a, nf = oracle.amax(x, cu, H, D, **src)
            qs, ds = self.rings[t].dynamic_step(a, nf)
            self.qs[t], self.ds[t] = qs, ds
        for t, x in enumerate(tensors_u16):
            codes.append(oracle.quantize(x, cu, H, D, self.qs[t], **src))
        return codes

    def set_static(self, A3):
        self.static = [np.float32(a) for a in A3]

    def static_pass(self, tensors_u16, cu, H, D=128, **src):
        codes = []
        for t, x in enumerate(tensors_u16):
            qs, ds = oracle.scales_from_bound(self.static[t])
            self.qs[t], self.ds[t] = qs, ds
            codes.append(oracle.quantize(x, cu, H, D, qs, **src))
        return codes


def bits(x: torch.Tensor) -> np.ndarray:
    return synthetic.bf16_bits(x)


def assert_codes_equal(got: torch.Tensor, want: np.ndarray, what: str = "codes"):
    g = got.cpu().numpy()
    if not np.array_equal(g, want):
        bad = np.argwhere(g != want)
        i = tuple(bad[0])
        raise AssertionError(f"{what}: {len(bad)} mismatches, first at {i}: "
                             f"got {g[i]:#04x} want {want[i]:#04x}")


def assert_scales_equal(ctx, layer, ol: OracleLayer):
    qs, ds = ctx.get_scales(layer)
    np.testing.assert_array_equal(qs, np.array(ol.qs, dtype=np.float32))
    np.testing.assert_array_equal(ds, np.array(ol.ds, dtype=np.float32))


def assert_ring_equal(ctx, layer, ol: OracleLayer):
    slots, meta = ctx.get_ring_state(layer)
    for t in range(3):
        r = ol.rings[t]
        assert meta[t, 0] == r.head and meta[t, 1] == r.count, (t, meta[t], r.head, r.count)
        np.testing.assert_array_equal(slots[t, :r.count], r.slots[:r.count])


def sample_rows(cu: np.ndarray, per_seq: int, seed: int = 0) -> np.ndarray:
    """Seeded query rows per sequence: first/last rows, tile edges, random."""
    rng = np.random.Generator(np.random.PCG64(seed))
    rows = []
    for b in range(len(cu) - 1):
        s0, s1 = int(cu[b]), int(cu[b + 1])
        n = s1 - s0
        if n == 0:
            continue
        pick = {0, n - 1, min(127, n - 1), min(128, n - 1), min(255, n - 1), min(256, n - 1),
                (n - 1) // 128 * 128, n // 2}
        k = max(0, min(per_seq, n) - len(pick))
        pick.update(rng.choice(n, size=min(k, n), replace=False).tolist())
        rows.extend(s0 + r for r in sorted(pick))
    return np.array(sorted(set(rows)), dtype=np.int64)


def attention_errors(got: torch.Tensor, want, rows: Optional[np.ndarray] = None):
    """(max, mean) of |got - ref| / max(1, |ref|).  `want` is the oracle output
    or an (output, ambiguity) pair; the ambiguity allowance (P codes within an
    fp32 evaluation's error of a rounding tie, where either neighbouring code
    is a correct result of the rule) is subtracted first, and outputs with an
    infinite allowance (a row whose reference-max move was decided at the
    threshold) are left out."""
    amb = np.zeros(1)
    if isinstance(want, tuple):
        want, amb = want
    g = got.float().cpu().numpy().astype(np.float64)
    if rows is not None:
        g = g[rows]
    amb = np.broadcast_to(amb, want.shape)
    keep = np.isfinite(amb)
    if not keep.any():
        return 0.0, 0.0
    d = np.maximum(np.abs(g - want)[keep] - amb[keep], 0.0) / np.maximum(1.0, np.abs(want[keep]))
    return float(d.max()), float(d.mean())


def assert_attention_close(got, want, rows=None, what="attention"):
    g = got.float().cpu().numpy()
    if rows is not None:
        g = g[rows]
    assert np.isfinite(g).all(), f"{what}: non-finite output"
    mx, mean = attention_errors(got, want, rows)
    ref = want[0] if isinstance(want, tuple) else want
    n_amb = int((want[1] > 0).sum()) if isinstance(want, tuple) else 0
    n_out = int(np.isinf(want[1]).sum()) if isinstance(want, tuple) else 0
    print(f"{what}: max|err| {mx:.3e} mean|err| {mean:.3e} (max|ref| {np.abs(ref).max():.3e}, "
          f"{n_amb} outputs with a tie allowance, {n_out} in rows decided at the threshold)")
    assert mx <= MAX_ABS_TOL and mean <= MEAN_ABS_TOL, (what, mx, mean)
    # threshold ties are rare; many of them would hide a wrong reference rule
    assert n_out <= max(2 * ref.shape[-1], ref.size // 100), (what, n_out)
    return mx, mean
