"""Shared helpers for the GPU parity tests: run the CUDA path through the
C-ABI binding, run the oracle on the same seeded inputs, compare."""
from __future__ import annotations

import math
from typing import Optional, Sequence, Tuple

import numpy as np
import torch

import oracle
import synthetic

# Attention tolerance against the oracle (fp64, same P rule): max abs error
# <= 1e-2 and mean abs error <= 1e-3.  Each output's error is the absolute
# difference less two allowances that no correct implementation can avoid:
# the oracle's tie allowance (P codes within the kernel's evaluation error of
# an E4M3 rounding tie, where either code is a correct result of the rule)
# and half a bf16 ulp of the output (the kernel's result is a bf16 value:
# RNE to bf16 moves it by up to half the spacing of bf16 numbers there).
MAX_ABS_TOL = 1e-2
MEAN_ABS_TOL = 1e-3
# Outputs of rows whose reference-max move was decided within the kernel's
# evaluation error of the threshold cannot be compared; more than this
# fraction of them would hide a wrong rule.
MAX_EXCLUDED_FRACTION = 1e-3

# Per-check records, printed as one table at the end of the session
# (tests/conftest.py), so they reach the log even when every check passes.
RECORDS = []


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
        # the first two query tiles' edges, every row of the last query block's
        # tile starts and ends (the ragged tail), and the middle
        pick = {0, n - 1, min(127, n - 1), min(128, n - 1), min(255, n - 1), min(256, n - 1),
                (n - 1) // 128 * 128, max(0, (n - 1) // 128 * 128 - 1), (n - 1) // 256 * 256,
                max(0, n - 129), n // 2}
        k = max(0, min(per_seq, n) - len(pick))
        pick.update(rng.choice(n, size=min(k, n), replace=False).tolist())
        rows.extend(s0 + r for r in sorted(pick))
    return np.array(sorted(set(rows)), dtype=np.int64)


def bf16_half_ulp(x: np.ndarray) -> np.ndarray:
    """Half the spacing of bf16 numbers at |x| (bf16 keeps 8 significant
    bits: spacing 2^(e-7) in [2^e, 2^(e+1)); subnormal spacing below 2^-126)."""
    a = np.abs(np.asarray(x, dtype=np.float64))
    a = np.where(np.isfinite(a), np.maximum(a, 2.0 ** -126), 2.0 ** 127)   # non-finite: any
    e = np.floor(np.log2(a))
    return np.ldexp(1.0, (e - 8).astype(np.int64))


def attention_errors(got: torch.Tensor, want, rows: Optional[np.ndarray] = None) -> dict:
    """Error statistics of a bf16 attention output against the oracle.

    ``want`` is the oracle's fp64 output or an (output, allowance) pair.
    Outputs where the oracle is not finite (a NaN or Inf input in the
    sequence's own Q/K/V) must be non-finite in ``got`` too and are not part
    of the statistics.  Returned keys: ``max``/``mean`` of the gated error
    max(0, |got - ref| - allowance - bf16_half_ulp), ``plain_max``/
    ``plain_mean`` of |got - ref| over the same outputs, ``n`` outputs
    compared, ``n_tie`` with a tie allowance, ``n_excluded`` in rows decided
    at the threshold, ``n_nonfinite_ok`` non-finite outputs that matched the
    oracle's, ``n_nonfinite_bad`` that did not, ``max_ref``."""
    amb = np.zeros(1)
    n_alt = 0
    if isinstance(want, tuple) and len(want) == 4:
        want, amb, alt, alt_amb = want
        g = got.float().cpu().numpy().astype(np.float64)
        if rows is not None:
            g = g[rows]
        # rows with two correct results (one reference move decided at the
        # threshold): compare each (row, head) with the result it is closer to
        has = np.isfinite(alt).all(axis=-1)
        if has.any():
            def worst(ref, a):
                e = np.abs(g - ref) - a - bf16_half_ulp(np.maximum(np.abs(ref), np.abs(g)))
                return np.where(np.isfinite(e), e, np.inf).max(axis=-1)
            pick = has & (worst(alt, alt_amb) < worst(want, amb))
            n_alt = int(pick.sum())
            want = np.where(pick[..., None], alt, want)
            amb = np.where(pick[..., None], alt_amb, amb)
        got = torch.from_numpy(g)
        rows = None
    elif isinstance(want, tuple):
        want, amb = want
    g = got.float().cpu().numpy().astype(np.float64)
    if rows is not None:
        g = g[rows]
    amb = np.broadcast_to(amb, want.shape)
    ref_finite = np.isfinite(want)
    n_nf_bad = int(np.sum(~ref_finite & np.isfinite(g)) + np.sum(ref_finite & ~np.isfinite(g)))
    n_nf_ok = int(np.sum(~ref_finite & ~np.isfinite(g)))
    excluded = ref_finite & ~np.isfinite(amb)
    keep = ref_finite & np.isfinite(amb) & np.isfinite(g)
    st = dict(n=int(keep.sum()), n_tie=int(((amb > 0) & keep).sum()), n_alt=n_alt,
              n_excluded=int(excluded.sum()), n_nonfinite_ok=n_nf_ok,
              n_nonfinite_bad=n_nf_bad, max=0.0, mean=0.0, plain_max=0.0, plain_mean=0.0,
              max_ref=float(np.abs(want[ref_finite]).max()) if ref_finite.any() else 0.0)
    if keep.any():
        gk, wk, ak = g[keep], want[keep], amb[keep]
        plain = np.abs(gk - wk)
        gated = np.maximum(plain - ak - bf16_half_ulp(np.maximum(np.abs(wk), np.abs(gk))), 0.0)
        st.update(max=float(gated.max()), mean=float(gated.mean()),
                  plain_max=float(plain.max()), plain_mean=float(plain.mean()))
    return st


def unquantized_errors(got: torch.Tensor, ref: np.ndarray, rows=None) -> Tuple[float, float]:
    """(max, mean) of |got - ref| against fp64 attention on the unquantised
    bf16 inputs: reported beside the parity figures, not gated."""
    g = got.float().cpu().numpy().astype(np.float64)
    if rows is not None:
        g = g[rows]
    d = np.abs(g - ref)
    d = d[np.isfinite(d)]
    return (float(d.max()), float(d.mean())) if d.size else (0.0, 0.0)


def assert_attention_close(got, want, rows=None, what="attention", unquantized=None):
    """Gate: gated max <= 1e-2, gated mean <= 1e-3, non-finite outputs where
    and only where the oracle's are, excluded outputs <= 0.1 %.  The figures
    go into the failure message and into the session summary.  With
    ``unquantized`` (fp64 attention on the bf16 inputs, same rows) the error
    against it is recorded too."""
    st = attention_errors(got, want, rows)
    total = st["n"] + st["n_excluded"]
    uq = unquantized_errors(got, unquantized, rows) if unquantized is not None else None
    RECORDS.append(dict(what=what, uq=uq, **st))
    msg = (f"{what}: gated max {st['max']:.3e} mean {st['mean']:.3e} | plain max "
           f"{st['plain_max']:.3e} mean {st['plain_mean']:.3e} | max|ref| {st['max_ref']:.3e} | "
           f"{st['n']} outputs, {st['n_tie']} with a tie allowance, {st['n_alt']} rows matched "
           f"against the other outcome of a move at the threshold, {st['n_excluded']} excluded "
           f"(two or more such moves), {st['n_nonfinite_ok']} non-finite as the oracle, "
           f"{st['n_nonfinite_bad']} non-finite mismatches")
    if uq is not None:
        msg += f" | vs unquantised fp64: max {uq[0]:.3e} mean {uq[1]:.3e}"
    print(msg)
    assert st["n_nonfinite_bad"] == 0, msg
    assert st["max"] <= MAX_ABS_TOL and st["mean"] <= MEAN_ABS_TOL, msg
    assert st["n_excluded"] <= MAX_EXCLUDED_FRACTION * max(total, 1), msg
    return st["max"], st["mean"]
