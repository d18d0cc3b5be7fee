"""CPU oracle for on-the-fly FP8 attention -- TEST INFRASTRUCTURE ONLY.

Only the tests, the smoke check and the benchmark's CPU-baseline leg may
import this package.  The product (the CUDA library and its Python binding)
never imports, links or calls it, and it shares no code with the product.

The arithmetic lives in ``fp8attn_oracle.c`` (plain C, fp64 attention, fp32
quantisation rules); this module only marshals numpy arrays.  Sources are the
pages on FP8 ViT/DiT attention quantisation:

* vLLM docs, "FP8 ViT encoder attention", usage section -- 16-entry amax
  ring driving the per-forward scale, static per-layer ``{q, k, v}`` scales,
  save margin (default 1.5), scale-file format section (``q_scale`` aliases).
* vLLM-Omni docs, "Quantized KV Cache", parameters table -- skip selectors:
  comma-separated integers and inclusive ranges.
* Ascend quantisation chapter -- FP8 formats E4M3 / E5M2 (names only).
"""
from __future__ import annotations

import ctypes
import math
import re
from typing import Iterable, Optional, Sequence

import numpy as np

from . import build_oracle

_lib = None

RING_LEN = 16          # vLLM FP8 ViT page: 16 observed amax values
DEFAULT_MARGIN = 1.5   # vLLM FP8 ViT page: --mm-encoder-fp8-scale-save-margin
E4M3_MAX = 448.0       # OCP E4M3 (FN) largest finite magnitude
P_SCALE = 32.0         # P is quantised as e4m3(32 exp(s - r)) (power of two: exact)
P_BLOCK = 128          # keys per P-quantisation block
P_LAG_LOG2 = 3.0       # the reference max r moves only when a block max exceeds it by more


class _Ring(ctypes.Structure):
    _fields_ = [("slot", ctypes.c_float * RING_LEN),
                ("head", ctypes.c_uint32),
                ("count", ctypes.c_uint32)]


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is not None:
        return _lib
    path = build_oracle.build()
    L = ctypes.CDLL(path)
    P = ctypes.c_void_p
    i64 = ctypes.c_int64
    i32 = ctypes.c_int
    f32 = ctypes.c_float
    f64 = ctypes.c_double
    L.or_e4m3_value.restype = f64
    L.or_e4m3_value.argtypes = [ctypes.c_uint8]
    L.or_e4m3_encode.restype = ctypes.c_uint8
    L.or_e4m3_encode.argtypes = [f64]
    L.or_e4m3_encode_f32_array.restype = None
    L.or_e4m3_encode_f32_array.argtypes = [P, i64, P]
    L.or_e4m3_value_array.restype = None
    L.or_e4m3_value_array.argtypes = [P, i64, P]
    L.or_amax_bf16.restype = f32
    L.or_amax_bf16.argtypes = [P, i64, i64, P, P, i32, i32, i32, ctypes.POINTER(i32), i32]
    L.or_quantize_bf16.restype = None
    L.or_quantize_bf16.argtypes = [P, i64, i64, P, P, i32, i32, i32, f32, P, i32]
    L.or_ring_reset.argtypes = [ctypes.POINTER(_Ring)]
    L.or_ring_push.argtypes = [ctypes.POINTER(_Ring), f32]
    L.or_ring_bound.restype = f32
    L.or_ring_bound.argtypes = [ctypes.POINTER(_Ring)]
    L.or_scales_from_bound.argtypes = [f32, ctypes.POINTER(f32), ctypes.POINTER(f32)]
    L.or_dynamic_step.argtypes = [ctypes.POINTER(_Ring), f32, i32,
                                  ctypes.POINTER(f32), ctypes.POINTER(f32)]
    L.or_export_value.restype = f32
    L.or_export_value.argtypes = [ctypes.POINTER(_Ring), f32]
    L.or_attention_fp8.restype = i32
    L.or_attention_fp8.argtypes = [P, P, P, P, i32, i32, i32, f64, f64, f64, f64,
                                   i32, i32, P, i64, P, P, P, P, i32]
    L.or_attention_bf16.restype = i32
    L.or_attention_bf16.argtypes = [P, P, P, P, i32, i32, i32, f64, P, i64, P, i32]
    _lib = L
    return L


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


# --------------------------------------------------------------------------
# E4M3
# --------------------------------------------------------------------------

def e4m3_value(codes) -> np.ndarray:
    """fp64 value of each E4M3 (FN) code (NaN for 0x7F / 0xFF)."""
    c = np.ascontiguousarray(np.asarray(codes, dtype=np.uint8))
    out = np.empty(c.shape, dtype=np.float64)
    lib().or_e4m3_value_array(_ptr(c), c.size, _ptr(out))
    return out


def e4m3_encode(y) -> np.ndarray:
    """E4M3 code of each value: RNE, ties to even, saturating, NaN -> 0x7F.

    ``y`` may be fp32 or fp64; fp32 inputs are encoded exactly as given."""
    y = np.asarray(y)
    if y.dtype == np.float32:
        y = np.ascontiguousarray(y)
        out = np.empty(y.shape, dtype=np.uint8)
        lib().or_e4m3_encode_f32_array(_ptr(y), y.size, _ptr(out))
        return out
    y = np.ascontiguousarray(y, dtype=np.float64)
    out = np.empty(y.shape, dtype=np.uint8)
    enc = lib().or_e4m3_encode
    flat_in, flat_out = y.reshape(-1), out.reshape(-1)
    for i in range(flat_in.size):
        flat_out[i] = enc(float(flat_in[i]))
    return out


def bf16_bits_to_f32(x_u16: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to fp32 (bit shift)."""
    return (np.asarray(x_u16, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


# --------------------------------------------------------------------------
# amax, cast (unpadding addressing: row t of sequence b reads source row t,
# or src_seq_start[b] + t - cu[b] for a padded source)
# --------------------------------------------------------------------------

def _tensor_args(x_u16, cu, H, D, tok_stride, head_stride, src_seq_start):
    x = np.ascontiguousarray(np.asarray(x_u16).view(np.uint16))
    cu = np.ascontiguousarray(np.asarray(cu, dtype=np.int32))
    B = cu.size - 1
    if tok_stride is None:
        tok_stride = H * D
    if head_stride is None:
        head_stride = D
    sss = None if src_seq_start is None else np.ascontiguousarray(
        np.asarray(src_seq_start, dtype=np.int32))
    return x, cu, B, int(tok_stride), int(head_stride), sss


def amax(x_u16, cu, H, D, tok_stride=None, head_stride=None, src_seq_start=None,
         nthreads: int = 0):
    """(amax, nonfinite): max |x| over valid tokens, NaN ignored."""
    x, cu, B, ts, hs, sss = _tensor_args(x_u16, cu, H, D, tok_stride, head_stride,
                                         src_seq_start)
    nf = ctypes.c_int(0)
    a = lib().or_amax_bf16(_ptr(x), ts, hs, _ptr(sss), _ptr(cu), B, H, D,
                           ctypes.byref(nf), nthreads)
    return np.float32(a), bool(nf.value)


def quantize(x_u16, cu, H, D, qs, tok_stride=None, head_stride=None,
             src_seq_start=None, nthreads: int = 0) -> np.ndarray:
    """Packed [T, H, D] E4M3 codes of fl32(x * qs)."""
    x, cu, B, ts, hs, sss = _tensor_args(x_u16, cu, H, D, tok_stride, head_stride,
                                         src_seq_start)
    T = int(cu[-1])
    out = np.empty((T, H, D), dtype=np.uint8)
    lib().or_quantize_bf16(_ptr(x), ts, hs, _ptr(sss), _ptr(cu), B, H, D,
                           float(np.float32(qs)), _ptr(out), nthreads)
    return out


# --------------------------------------------------------------------------
# Ring and scales
# --------------------------------------------------------------------------

def scales_from_bound(A) -> tuple:
    """(qs, ds) = (fl32(448/A), fl32(A/448)); A == 0 gives (1, 1)."""
    qs, ds = ctypes.c_float(), ctypes.c_float()
    lib().or_scales_from_bound(float(np.float32(A)), ctypes.byref(qs), ctypes.byref(ds))
    return np.float32(qs.value), np.float32(ds.value)


class Ring:
    """16-entry circular buffer of observed amax values for one tensor."""

    def __init__(self):
        self._r = _Ring()
        lib().or_ring_reset(ctypes.byref(self._r))

    @property
    def slots(self) -> np.ndarray:
        return np.array(self._r.slot[:], dtype=np.float32)

    @property
    def head(self) -> int:
        return int(self._r.head)

    @property
    def count(self) -> int:
        return int(self._r.count)

    def push(self, amax_value) -> None:
        lib().or_ring_push(ctypes.byref(self._r), float(np.float32(amax_value)))

    def bound(self) -> np.float32:
        return np.float32(lib().or_ring_bound(ctypes.byref(self._r)))

    def dynamic_step(self, amax_value, nonfinite: bool = False) -> tuple:
        """Push the current amax (unless non-finite), then scales from the bound."""
        qs, ds = ctypes.c_float(), ctypes.c_float()
        lib().or_dynamic_step(ctypes.byref(self._r), float(np.float32(amax_value)),
                              int(bool(nonfinite)), ctypes.byref(qs), ctypes.byref(ds))
        return np.float32(qs.value), np.float32(ds.value)

    def export_value(self, margin: float = DEFAULT_MARGIN) -> np.float32:
        """fl32(bound * margin): the value written to the static scale map."""
        return np.float32(lib().or_export_value(ctypes.byref(self._r),
                                                float(np.float32(margin))))


# --------------------------------------------------------------------------
# Attention
# --------------------------------------------------------------------------

def _rows_arg(rows):
    if rows is None:
        return None, 0
    r = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    return r, r.size


P_LINEAR_LOG, P_EXP2 = "linear_log", "exp2"


def attention_fp8(q8, k8, v8, cu, ds_qkv: Sequence[float], scale: Optional[float] = None,
                  pquant: bool = True, l_of_quantized: bool = False, rows=None,
                  nthreads: int = 0, return_ambiguity: bool = False, rule: str = P_LINEAR_LOG,
                  return_alternative: bool = False):
    """fp64 attention on E4M3 codes [T, H, D]; returns [len(rows) or T, H, D].

    With ``pquant`` the PV product uses P quantised per block of 128 keys (in
    sequence order) as e4m3(32 exp(s - r))/32 against the row's reference max
    r: block 0's max, replaced by a later block's max only when that exceeds
    r by more than 3 in log2 units; each block is carried exactly to the final
    max M; l is the sum of the unquantised exp(s - M) unless
    ``l_of_quantized``.

    ``rule`` selects the quantisation of each block's P (both against the
    same lagged reference r, t = (s - r) log2(e) + 5):
    ``"exp2"``: code = e4m3(2^t) (RNE), l from the unquantised values as
    above; ``"linear_log"``: code = 8 t + 56 rounded to the nearest integer
    (ties to even) and clamped to [0, 128] -- the E4M3 bit pattern read as a
    fixed-point log2, i.e. the piecewise-linear interpolation of 2^t between
    powers of two rounded to the E4M3 grid -- with l the sum of the
    quantised values and code 0 for NaN scores.

    With ``return_ambiguity`` also returns, per output, the largest change
    that P codes lying within an fp32 evaluation's error of a rounding tie
    can make (either neighbouring code is a correct result there), and +inf
    for every output of a row whose reference-max move was decided within
    such an error of the threshold (that row cannot be compared).

    With ``return_alternative`` (implies ``return_ambiguity``) a row whose
    reference moves exactly once within that error of the threshold is not
    given up: it is evaluated both ways, and the second result and its
    allowance come back as two more arrays (NaN for rows with one result);
    only rows with two or more such decisions keep the infinite allowance."""
    q8 = np.ascontiguousarray(q8, dtype=np.uint8)
    k8 = np.ascontiguousarray(k8, dtype=np.uint8)
    v8 = np.ascontiguousarray(v8, dtype=np.uint8)
    T, H, D = q8.shape
    cu = np.ascontiguousarray(np.asarray(cu, dtype=np.int32))
    if rule not in (P_LINEAR_LOG, P_EXP2):
        raise ValueError(f"unknown P rule {rule!r}")
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    r, nr = _rows_arg(rows)
    n = nr if r is not None else int(cu[-1])
    out = np.empty((n, H, D), dtype=np.float64)
    return_ambiguity = return_ambiguity or return_alternative
    amb = np.empty((n, H, D), dtype=np.float64) if return_ambiguity else None
    alt = np.empty((n, H, D), dtype=np.float64) if return_alternative else None
    alt_amb = np.empty((n, H, D), dtype=np.float64) if return_alternative else None
    lib().or_attention_fp8(_ptr(q8), _ptr(k8), _ptr(v8), _ptr(cu), cu.size - 1, H, D,
                           float(ds_qkv[0]), float(ds_qkv[1]), float(ds_qkv[2]),
                           float(scale), (2 if rule == P_LINEAR_LOG else 1) if pquant else 0,
                           int(bool(l_of_quantized)),
                           _ptr(r), nr, _ptr(out), _ptr(amb), _ptr(alt), _ptr(alt_amb), nthreads)
    if return_alternative:
        return out, amb, alt, alt_amb
    return (out, amb) if return_ambiguity else out


def attention_bf16(q_u16, k_u16, v_u16, cu, scale: Optional[float] = None, rows=None,
                   nthreads: int = 0) -> np.ndarray:
    """fp64 attention on bf16 inputs [T, H, D] (skip-layer path, no quantisation)."""
    q = np.ascontiguousarray(np.asarray(q_u16).view(np.uint16))
    k = np.ascontiguousarray(np.asarray(k_u16).view(np.uint16))
    v = np.ascontiguousarray(np.asarray(v_u16).view(np.uint16))
    T, H, D = q.shape
    cu = np.ascontiguousarray(np.asarray(cu, dtype=np.int32))
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    r, nr = _rows_arg(rows)
    n = nr if r is not None else int(cu[-1])
    out = np.empty((n, H, D), dtype=np.float64)
    lib().or_attention_bf16(_ptr(q), _ptr(k), _ptr(v), _ptr(cu), cu.size - 1, H, D,
                            float(scale), _ptr(r), nr, _ptr(out), nthreads)
    return out


# --------------------------------------------------------------------------
# Host logic: selectors, modes, calibrate-then-serve
# --------------------------------------------------------------------------

_SEL_ITEM = re.compile(r"^\s*(\d+)\s*(?:-\s*(\d+)\s*)?$")


def parse_selector(text: Optional[str], max_index: int) -> set:
    """Indices named by a selector: comma-separated integers and inclusive
    ranges ("0,1,4-6").  Empty or None names nothing.  Raises ValueError for
    malformed items, reversed ranges or indices >= max_index."""
    if text is None or text.strip() == "":
        return set()
    out = set()
    for item in text.split(","):
        m = _SEL_ITEM.match(item)
        if not m:
            raise ValueError(f"malformed selector item {item!r}")
        lo = int(m.group(1))
        hi = int(m.group(2)) if m.group(2) is not None else lo
        if hi < lo or hi >= max_index:
            raise ValueError(f"selector item {item!r} out of range")
        out.update(range(lo, hi + 1))
    return out


DYNAMIC, STATIC, SKIP = 0, 1, 2


def layer_mode(layer: int, skip: Iterable[int], has_static: bool) -> int:
    """SKIP for selected layers, STATIC once static scales are set, else DYNAMIC."""
    if layer in set(skip):
        return SKIP
    return STATIC if has_static else DYNAMIC


def step_layer_mode(layer: int, step: int, skip_layers: Iterable[int], skip_steps: Iterable[int],
                    has_static: bool) -> int:
    """vLLM-Omni parameters table (kv_cache_skip_steps, kv_cache_skip_layers):
    listed denoising steps or layers keep the native dtype (SKIP); every other
    call uses the FP8 path, STATIC once static scales are set, else DYNAMIC."""
    if step in set(skip_steps):
        return SKIP
    return layer_mode(layer, skip_layers, has_static)
