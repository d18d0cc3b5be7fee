"""fp8attn for B200 (sm_100a): on-the-fly FP8 (E4M3) quantisation of Q/K/V
with per-tensor scales from a device-resident 16-entry amax ring or from
static per-layer bounds, and a varlen non-causal FP8 flash-attention forward
on tcgen05 tensor cores.

This module is a thin ctypes binding over ``libfp8attn.so`` (built from
``csrc/`` by ``build.py``): it only marshals torch tensors into device
pointers, sizes and streams.  Every step of the path runs in the library's
CUDA kernels; there is no CPU or PyTorch fallback, and every call fails
loudly if the library is missing or no CUDA device is present.

Names follow the C ABI in ``include/fp8attn.h`` without the ``fp8attn_``
prefix.
"""
from __future__ import annotations

import contextlib
import ctypes
import math
import os
from typing import Dict, Iterable, List, Optional, Sequence, Tuple

import numpy as np
import torch

__all__ = [
    "DYNAMIC", "STATIC", "SKIP", "P_LINEAR_LOG", "P_EXP2", "RING_LENGTH", "DEFAULT_MARGIN", "FP8AttnError", "lib",
    "Context", "varlen_fwd", "varlen_fwd_bf16", "parse_selector", "e4m3_encode",
    "launch_count", "load_scale_file", "save_scale_file", "apply_margin", "read_error_word",
    "quantize_qkv_noalloc", "quantize_qkv_noalloc_error", "RING",
    "head_sharded_dynamic_quantize", "regroup_heads", "TorchComm", "ulysses_attention",
]

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libfp8attn.so")

DYNAMIC, STATIC, SKIP, RING = 0, 1, 2, 3
P_LINEAR_LOG, P_EXP2 = 0, 1
# work schedules of the FP8 attention kernel (fp8attn_schedule in fp8attn.h)
SCHED_AUTO, SCHED_WHOLE, SCHED_SPLIT = 0, 1, 2
RING_LENGTH = 16
DEFAULT_MARGIN = 1.5
HEAD_DIM = 128

_STATUS = {
    0: "ok", 1: "invalid argument", 2: "CUDA error", 3: "device wait timed out",
    4: "unsupported configuration", 5: "non-finite amax", 6: "inconsistent cu_seqlens",
}


class FP8AttnError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {_STATUS.get(status, 'status %d' % status)}")


_lib: Optional[ctypes.CDLL] = None


def lib() -> ctypes.CDLL:
    """Load ``libfp8attn.so`` (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(
            f"{LIB_PATH} is missing: build it with "
            "`python -m quantization_amax_reduce_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    P, I, I64, F, U8P = (ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float,
                         ctypes.c_void_p)
    sigs = {
        "fp8attn_status_string": (ctypes.c_char_p, [I]),
        "fp8attn_ring_length": (I, []),
        "fp8attn_workspace_bytes": (ctypes.c_size_t, [I]),
        "fp8attn_create": (I, [I, P, ctypes.c_size_t, P, ctypes.POINTER(P)]),
        "fp8attn_destroy": (I, [P]),
        "fp8attn_quantize_qkv": (I, [P, I, I, P, P, P, I64, I64, P, P, I, I, I64, I, I, P, P, P,
                                     P]),
        "fp8attn_quantize_qkv_grouped": (I, [P, I, I, P, P, P, I64, I64, P, P, I, I, I64, I, I, I,
                                             P, P, P, P]),
        "fp8attn_amax_ring_update": (I, [P, I, P, P]),
        "fp8attn_amax_qkv": (I, [P, P, P, P, I64, I64, P, P, I, I, I64, I, I, P, P]),
        "fp8attn_set_static_scales": (I, [P, I, F, F, F, P]),
        "fp8attn_clear_static_scales": (I, [P, I]),
        "fp8attn_has_static_scales": (I, [P, I]),
        "fp8attn_export_static_scales": (I, [P, F, P, P]),
        "fp8attn_descale_ptr": (P, [P, I]),
        "fp8attn_quant_scale_ptr": (P, [P, I]),
        "fp8attn_get_ring_state": (I, [P, I, P, P, P]),
        "fp8attn_set_ring_state": (I, [P, I, P, P, P]),
        "fp8attn_get_scales": (I, [P, I, P, P]),
        "fp8attn_varlen_fwd": (I, [P, P, P, P, I, I, I64, I, I, P, F, P, P, P]),
        "fp8attn_varlen_fwd_rule": (I, [P, P, P, P, I, I, I64, I, I, P, F, I, P, P, P]),
        "fp8attn_varlen_fwd_sched": (I, [P, P, P, P, I, I, I64, I, I, P, F, I, I, P, P, P]),
        "fp8attn_varlen_fwd_bf16": (I, [P, P, P, P, I, I, I64, I, I, F, P, P, P]),
        "fp8attn_varlen_fwd_static": (I, [P, I, P, P, P, I64, I64, P, I, I, I64, I, I, F, I, P,
                                          P]),
        "fp8attn_get_error": (I, [P, P]),
        "fp8attn_read_error_word": (I, [P, P]),
        "fp8attn_parse_selector": (I, [ctypes.c_char_p, I, U8P]),
        "fp8attn_select_mode": (I, [P, U8P, I]),
        "fp8attn_select_mode_at_step": (I, [P, U8P, I, U8P, I, I]),
        "fp8attn_e4m3_encode": (I, [P, I64, F, P, P]),
        "fp8attn_launch_count": (ctypes.c_uint64, []),
        "fp8attn_quantize_qkv_noalloc": (I, [P, P, P, I64, I64, P, P, I, I, I64, I, I, P, P, P, P,
                                             P, P]),
        "fp8attn_quantize_qkv_noalloc_error": (I, [P]),
        "fp8attn_selftest_bounded_waits": (I, [ctypes.c_uint64, ctypes.POINTER(I), P]),
        "fp8attn_regroup_heads": (I, [P, P, I64, I, I, I, I, P]),
        "fp8attn_selftest_qk_scores": (I, [P, P, I64, P, P, P]),
        "fp8attn_apply_margin": (I, [P, I64, F, P]),
        "fp8attn_scale_map_parse": (I, [ctypes.c_char_p, ctypes.c_size_t, F, I, P, P,
                                        ctypes.POINTER(I)]),
        "fp8attn_scale_map_format": (I, [I, P, P, P, ctypes.c_size_t,
                                         ctypes.POINTER(ctypes.c_size_t)]),
    }
    for name, (res, args) in sigs.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    _lib = L
    return L


def _check(status: int, what: str) -> None:
    if status != 0:
        raise FP8AttnError(status, what)


def _require_cuda(t: torch.Tensor, name: str) -> None:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")


def _stream(stream, device) -> int:
    if stream is None:
        return torch.cuda.current_stream(device).cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _qkv_source(q, k, v, cu_seqlens, total_tokens, src_seq_start):
    """Checks shared by the quantisation entry points; returns (H, tok_stride,
    head_stride, cu, B, total_tokens, src_seq_start tensor or None)."""
    for name, t in (("q", q), ("k", k), ("v", v)):
        _require_cuda(t, name)
        if t.dtype != torch.bfloat16:
            raise ValueError(f"{name} must be bfloat16")
    if q.shape != k.shape or q.shape != v.shape or q.stride() != k.stride() or \
            q.stride() != v.stride():
        raise ValueError("q, k, v must share shape and strides")
    if q.shape[-1] != HEAD_DIM or q.stride(-1) != 1:
        raise ValueError("head_dim must be 128 and contiguous")
    if q.dim() not in (3, 4):
        raise ValueError("sources are [T, H, 128] or [B, S_max, H, 128]")
    if q.dim() == 4 and q.shape[0] > 1 and q.stride(0) != q.shape[1] * q.stride(1):
        # the kernels address row r of a padded source at r * tok_stride
        raise ValueError("a padded source needs its sequences back to back "
                         "(stride(0) == S_max * stride(1))")
    H = q.shape[-2]
    head_stride, tok_stride = q.stride(-2), q.stride(-3)
    rows = q.shape[-3] if q.dim() == 3 else q.shape[0] * q.shape[1]
    if src_seq_start is not None and not isinstance(src_seq_start, torch.Tensor) and \
            not isinstance(cu_seqlens, torch.Tensor):
        _check_padded_rows(cu_seqlens, src_seq_start, rows)
    cu = _cu_tensor(cu_seqlens, q.device)
    B = cu.numel() - 1
    if total_tokens is None:
        if src_seq_start is not None:
            raise ValueError("total_tokens is required with a padded source")
        total_tokens = rows
    elif src_seq_start is None and int(total_tokens) > rows:
        raise ValueError(f"total_tokens {total_tokens} exceeds the {rows} source rows")
    sss = None
    if src_seq_start is not None:
        sss = _cu_tensor(src_seq_start, q.device)
    return H, tok_stride, head_stride, cu, B, total_tokens, sss


def _check_padded_rows(cu_seqlens, src_seq_start, rows: int) -> None:
    """Host-side check of a padded source given as host arrays: sequence b's
    rows [src_seq_start[b], src_seq_start[b] + len_b) lie inside the source's
    ``rows`` rows.  (Device tensors are not read back; the kernels take them
    as given.)"""
    cu = np.asarray(cu_seqlens, dtype=np.int64).ravel()
    start = np.asarray(src_seq_start, dtype=np.int64).ravel()
    if start.size != cu.size - 1:
        raise ValueError("src_seq_start needs one entry per sequence")
    lens = np.diff(cu)
    if (lens < 0).any():
        raise ValueError("cu_seqlens must not decrease")
    if (start < 0).any() or (start + lens > rows).any():
        raise ValueError(f"a sequence of the padded source lies outside its {rows} rows")


def _check_out(t, name: str, dtype, numel: int, device) -> None:
    """A caller-provided output: contiguous, on the inputs' device, of the
    right dtype and large enough that no kernel writes past its end."""
    _require_cuda(t, name)
    if t.dtype != dtype or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous {dtype} tensor")
    if t.device != torch.device(device):
        raise ValueError(f"{name} must be on {device}")
    if t.numel() < numel:
        raise ValueError(f"{name} holds {t.numel()} elements, {numel} needed")


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _cu_tensor(cu, device) -> torch.Tensor:
    if isinstance(cu, torch.Tensor):
        if cu.dtype != torch.int32 or not cu.is_cuda:
            raise ValueError("cu_seqlens must be an int32 CUDA tensor")
        return cu
    return torch.as_tensor(np.asarray(cu, dtype=np.int32), device=device)


# ---------------------------------------------------------------------------
# context: device-resident rings and scales
# ---------------------------------------------------------------------------

class Context:
    """Per-model scale state (one amax ring + scales per attention layer).

    The device workspace is a torch allocation owned by this object."""

    def __init__(self, num_layers: int, device=None, stream=None):
        L = lib()
        self.device = torch.device(device if device is not None else "cuda")
        if self.device.type != "cuda":
            raise ValueError("Context needs a CUDA device")
        self.num_layers = int(num_layers)
        nbytes = L.fp8attn_workspace_bytes(self.num_layers)
        if nbytes == 0:
            raise ValueError("num_layers must be >= 1")
        with torch.cuda.device(self.device):
            self.workspace = torch.empty(nbytes, dtype=torch.uint8, device=self.device)
            h = ctypes.c_void_p()
            _check(L.fp8attn_create(self.num_layers, _ptr(self.workspace), nbytes,
                                    ctypes.c_void_p(_stream(stream, self.device)),
                                    ctypes.byref(h)), "fp8attn_create")
        self._h = h

    def __del__(self):
        h = getattr(self, "_h", None)
        if h is not None and h.value and _lib is not None:
            _lib.fp8attn_destroy(h)
            self._h = None

    # -- hot path ---------------------------------------------------------
    def quantize_qkv(self, layer: int, mode: int, q: torch.Tensor, k: torch.Tensor,
                     v: torch.Tensor, cu_seqlens, max_seqlen: int, *,
                     total_tokens: Optional[int] = None, src_seq_start=None,
                     out: Optional[Sequence[torch.Tensor]] = None, stream=None
                     ) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
        """Fused amax + ring/scale update + E4M3 cast + unpad of one layer's
        Q, K, V.  Sources are bf16 with the channel contiguous: packed
        [T, H, 128], padded [B, S_max, H, 128] (pass ``src_seq_start``), or any
        strided view (e.g. slices of a fused [T, 3, H, 128] projection).
        Returns packed uint8 E4M3 codes [T, H, 128].  Mode RING casts with the
        layer's current ring scales (the cast step of a head-sharded pass)."""
        H, tok_stride, head_stride, cu, B, total_tokens, sss = _qkv_source(
            q, k, v, cu_seqlens, total_tokens, src_seq_start)
        if out is None:
            out = [torch.empty((total_tokens, H, HEAD_DIM), dtype=torch.uint8, device=q.device)
                   for _ in range(3)]
        else:
            if len(out) != 3:
                raise ValueError("out must hold three tensors (q8, k8, v8)")
            for name, t in zip(("q8", "k8", "v8"), out):
                _check_out(t, name, torch.uint8, int(total_tokens) * H * HEAD_DIM, q.device)
        _check(lib().fp8attn_quantize_qkv(
            self._h, layer, mode, _ptr(q), _ptr(k), _ptr(v), tok_stride, head_stride, _ptr(sss),
            _ptr(cu), B, int(max_seqlen), int(total_tokens), H, HEAD_DIM, _ptr(out[0]),
            _ptr(out[1]), _ptr(out[2]), ctypes.c_void_p(_stream(stream, q.device))),
            "fp8attn_quantize_qkv")
        return out[0], out[1], out[2]

    def varlen_fwd_static(self, layer: int, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                          cu_seqlens, max_seqlen: int, *, softmax_scale: float = 0.0,
                          total_tokens: Optional[int] = None, out: Optional[torch.Tensor] = None,
                          stream=None, p_rule: int = P_LINEAR_LOG) -> torch.Tensor:
        """Static-scale quantisation and FP8 attention in one launch: bit for
        bit ``varlen_fwd(*quantize_qkv(layer, STATIC, q, k, v, ...), ...,
        descale_ptr(layer))`` without the E4M3 copies in device memory.
        Sources are packed bf16 [T, H, 128] or a strided view of that shape
        (e.g. slices of a fused [T, 3, H, 128] projection); returns bf16
        [T, H, 128].  Device-side errors go to the context (``get_error``)."""
        if q.dim() != 3:
            raise ValueError("sources are packed [T, H, 128] (no padded layout)")
        H, tok_stride, head_stride, cu, B, total_tokens, _ = _qkv_source(
            q, k, v, cu_seqlens, total_tokens, None)
        dev = self.workspace.device          # the context's concrete device
        if q.device != dev or cu.device != dev:
            # the kernel reads the context's scales from its device workspace
            raise ValueError(f"q, k, v and cu_seqlens must be on the context's {dev}")
        n = int(total_tokens) * H * HEAD_DIM
        if out is None:
            out = torch.empty((total_tokens, H, HEAD_DIM), dtype=torch.bfloat16, device=q.device)
        else:
            _check_out(out, "out", torch.bfloat16, n, q.device)
        with torch.cuda.device(dev):
            _check(lib().fp8attn_varlen_fwd_static(
                self._h, layer, _ptr(q), _ptr(k), _ptr(v), tok_stride, head_stride, _ptr(cu), B,
                int(max_seqlen), int(total_tokens), H, HEAD_DIM, float(softmax_scale),
                int(p_rule), _ptr(out), ctypes.c_void_p(_stream(stream, q.device))),
                "fp8attn_varlen_fwd_static")
        return out

    def quantize_qkv_grouped(self, layer: int, mode: int, q: torch.Tensor, k: torch.Tensor,
                             v: torch.Tensor, cu_seqlens, max_seqlen: int, groups: int, *,
                             total_tokens: Optional[int] = None, src_seq_start=None,
                             out=None, stream=None
                             ) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
        """The STATIC or RING cast of ``quantize_qkv`` written head-grouped:
        returns uint8 E4M3 codes [groups, T, H / groups, 128] per tensor, group
        g holding heads [g H/groups, (g+1) H/groups) -- the send buffers of a
        sequence-parallel all-to-all, in one launch."""
        H, tok_stride, head_stride, cu, B, total_tokens, sss = _qkv_source(
            q, k, v, cu_seqlens, total_tokens, src_seq_start)
        groups = int(groups)
        if groups < 1 or H % groups:
            raise ValueError(f"groups {groups} must divide the {H} heads")
        if out is None:
            out = [torch.empty((groups, total_tokens, H // groups, HEAD_DIM), dtype=torch.uint8,
                               device=q.device) for _ in range(3)]
        else:
            if len(out) != 3:
                raise ValueError("out must hold three tensors (q8, k8, v8)")
            for name, t in zip(("q8", "k8", "v8"), out):
                _check_out(t, name, torch.uint8, int(total_tokens) * H * HEAD_DIM, q.device)
        _check(lib().fp8attn_quantize_qkv_grouped(
            self._h, layer, mode, _ptr(q), _ptr(k), _ptr(v), tok_stride, head_stride, _ptr(sss),
            _ptr(cu), B, int(max_seqlen), int(total_tokens), H, HEAD_DIM, groups, _ptr(out[0]),
            _ptr(out[1]), _ptr(out[2]), ctypes.c_void_p(_stream(stream, q.device))),
            "fp8attn_quantize_qkv_grouped")
        return out[0], out[1], out[2]

    def amax_qkv(self, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, cu_seqlens,
                 max_seqlen: int, *, total_tokens: Optional[int] = None, src_seq_start=None,
                 out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
        """Per-tensor amax (q, k, v) over the valid tokens into a device fp32
        [3] tensor; nothing is cast and no ring changes (sources as
        quantize_qkv)."""
        H, tok_stride, head_stride, cu, B, total_tokens, sss = _qkv_source(
            q, k, v, cu_seqlens, total_tokens, src_seq_start)
        if out is None:
            out = torch.empty(3, dtype=torch.float32, device=q.device)
        else:
            _check_out(out, "out", torch.float32, 3, q.device)
        _check(lib().fp8attn_amax_qkv(
            self._h, _ptr(q), _ptr(k), _ptr(v), tok_stride, head_stride, _ptr(sss), _ptr(cu), B,
            int(max_seqlen), int(total_tokens), H, HEAD_DIM, _ptr(out),
            ctypes.c_void_p(_stream(stream, q.device))), "fp8attn_amax_qkv")
        return out

    def amax_ring_update(self, layer: int, amax3: torch.Tensor, stream=None) -> None:
        """Push three device-side fp32 amax values (q, k, v) into the rings."""
        _require_cuda(amax3, "amax3")
        if amax3.dtype != torch.float32 or amax3.numel() != 3:
            raise ValueError("amax3 must be 3 fp32 values")
        _check(lib().fp8attn_amax_ring_update(self._h, layer, _ptr(amax3.contiguous()),
                                              ctypes.c_void_p(_stream(stream, self.device))),
               "fp8attn_amax_ring_update")

    def set_static_scales(self, layer: int, q: float, k: float, v: float, stream=None) -> None:
        _check(lib().fp8attn_set_static_scales(self._h, layer, float(q), float(k), float(v),
                                               ctypes.c_void_p(_stream(stream, self.device))),
               "fp8attn_set_static_scales")

    def clear_static_scales(self, layer: int) -> None:
        _check(lib().fp8attn_clear_static_scales(self._h, layer), "fp8attn_clear_static_scales")

    def has_static_scales(self, layer: int) -> bool:
        r = lib().fp8attn_has_static_scales(self._h, layer)
        if r < 0:
            raise FP8AttnError(1, "fp8attn_has_static_scales")
        return bool(r)

    def export_static_scales(self, margin: float = DEFAULT_MARGIN, stream=None) -> np.ndarray:
        """[num_layers, 3] float32: fl32(max(ring) * margin) per layer and tensor."""
        out = np.zeros((self.num_layers, 3), dtype=np.float32)
        _check(lib().fp8attn_export_static_scales(
            self._h, float(margin), out.ctypes.data_as(ctypes.c_void_p),
            ctypes.c_void_p(_stream(stream, self.device))), "fp8attn_export_static_scales")
        return out

    def descale_ptr(self, layer: int) -> int:
        p = lib().fp8attn_descale_ptr(self._h, layer)
        if not p:
            raise FP8AttnError(1, "fp8attn_descale_ptr")
        return int(p)

    def quant_scale_ptr(self, layer: int) -> int:
        p = lib().fp8attn_quant_scale_ptr(self._h, layer)
        if not p:
            raise FP8AttnError(1, "fp8attn_quant_scale_ptr")
        return int(p)

    def get_ring_state(self, layer: int, stream=None) -> Tuple[np.ndarray, np.ndarray]:
        slots = np.zeros((3, RING_LENGTH), dtype=np.float32)
        meta = np.zeros((3, 2), dtype=np.uint32)
        _check(lib().fp8attn_get_ring_state(self._h, layer, slots.ctypes.data_as(ctypes.c_void_p),
                                            meta.ctypes.data_as(ctypes.c_void_p),
                                            ctypes.c_void_p(_stream(stream, self.device))),
               "fp8attn_get_ring_state")
        return slots, meta

    def set_ring_state(self, layer: int, slots: np.ndarray, meta: np.ndarray, stream=None) -> None:
        s = np.ascontiguousarray(slots, dtype=np.float32).reshape(3, RING_LENGTH)
        m = np.ascontiguousarray(meta, dtype=np.uint32).reshape(3, 2)
        _check(lib().fp8attn_set_ring_state(self._h, layer, s.ctypes.data_as(ctypes.c_void_p),
                                            m.ctypes.data_as(ctypes.c_void_p),
                                            ctypes.c_void_p(_stream(stream, self.device))),
               "fp8attn_set_ring_state")

    def get_scales(self, layer: int, stream=None) -> Tuple[np.ndarray, np.ndarray]:
        """(qs[3], ds[3]) currently held for the layer."""
        out = np.zeros(6, dtype=np.float32)
        _check(lib().fp8attn_get_scales(self._h, layer, out.ctypes.data_as(ctypes.c_void_p),
                                        ctypes.c_void_p(_stream(stream, self.device))),
               "fp8attn_get_scales")
        return out[:3].copy(), out[3:].copy()

    def get_error(self, stream=None) -> int:
        """Read and clear the device error word; returns the status code."""
        return int(lib().fp8attn_get_error(self._h, ctypes.c_void_p(_stream(stream, self.device))))

    def select_mode(self, layer: int, skip_mask: Optional[np.ndarray] = None) -> int:
        m = None
        if skip_mask is not None:
            m = np.ascontiguousarray(skip_mask, dtype=np.uint8)
        r = lib().fp8attn_select_mode(self._h, None if m is None else m.ctypes.data_as(ctypes.c_void_p),
                                      layer)
        if r < 0:
            raise FP8AttnError(1, "fp8attn_select_mode")
        return r

    def select_mode_at_step(self, layer: int, step: int, skip_layers: Optional[np.ndarray] = None,
                            skip_steps: Optional[np.ndarray] = None) -> int:
        """Mode of layer `layer` at denoising step `step`: SKIP if either mask
        selects it, else STATIC/DYNAMIC as select_mode."""
        ml = None if skip_layers is None else np.ascontiguousarray(skip_layers, dtype=np.uint8)
        ms = None if skip_steps is None else np.ascontiguousarray(skip_steps, dtype=np.uint8)
        r = lib().fp8attn_select_mode_at_step(
            self._h, None if ml is None else ml.ctypes.data_as(ctypes.c_void_p), layer,
            None if ms is None else ms.ctypes.data_as(ctypes.c_void_p),
            0 if ms is None else int(ms.size), step)
        if r < 0:
            raise FP8AttnError(1, "fp8attn_select_mode_at_step")
        return r


# ---------------------------------------------------------------------------
# attention
# ---------------------------------------------------------------------------

def _attn_common(q, k, v, cu_seqlens, out, dtype):
    for name, t in (("q", q), ("k", k), ("v", v)):
        _require_cuda(t, name)
        if t.dtype != dtype or not t.is_contiguous() or t.dim() != 3 or t.shape[-1] != HEAD_DIM:
            raise ValueError(f"{name} must be a contiguous [T, H, 128] {dtype} tensor")
    if q.shape != k.shape or q.shape != v.shape:
        raise ValueError("q, k, v must have the same shape")
    T, H, _ = q.shape
    cu = _cu_tensor(cu_seqlens, q.device)
    if out is None:
        out = torch.empty((T, H, HEAD_DIM), dtype=torch.bfloat16, device=q.device)
    else:
        _check_out(out, "out", torch.bfloat16, T * H * HEAD_DIM, q.device)
    return T, H, cu, out


def varlen_fwd(q8: torch.Tensor, k8: torch.Tensor, v8: torch.Tensor, cu_seqlens,
               max_seqlen: int, descale, softmax_scale: float = 0.0,
               out: Optional[torch.Tensor] = None, error: Optional[torch.Tensor] = None,
               stream=None, p_rule: int = P_LINEAR_LOG,
               schedule: int = SCHED_AUTO) -> torch.Tensor:
    """FP8 attention on packed E4M3 [T, H, 128] codes.  ``descale`` is a device
    pointer (int, e.g. ``Context.descale_ptr(layer)``) or a 3-element fp32 CUDA
    tensor {ds_q, ds_k, ds_v}.  ``p_rule`` picks how P is quantised for the PV
    product (P_LINEAR_LOG, the default, or P_EXP2; see fp8attn_p_rule in
    fp8attn.h); ``schedule`` how the work units are laid on the GPU
    (SCHED_AUTO, SCHED_WHOLE or SCHED_SPLIT; bit-identical results, see
    fp8attn_schedule).
    Returns bf16 [T, H, 128]."""
    T, H, cu, out = _attn_common(q8, k8, v8, cu_seqlens, out, torch.uint8)
    if isinstance(descale, torch.Tensor):
        _require_cuda(descale, "descale")
        if descale.dtype != torch.float32 or descale.numel() != 3 or not descale.is_contiguous():
            raise ValueError("descale must be 3 contiguous fp32 values")
        dptr = ctypes.c_void_p(descale.data_ptr())
    else:
        dptr = ctypes.c_void_p(int(descale))
    _check(lib().fp8attn_varlen_fwd_sched(_ptr(q8), _ptr(k8), _ptr(v8), _ptr(cu), cu.numel() - 1,
                                          int(max_seqlen), T, H, HEAD_DIM, dptr,
                                          float(softmax_scale), int(p_rule), int(schedule),
                                          _ptr(out), _ptr(error),
                                          ctypes.c_void_p(_stream(stream, q8.device))),
           "fp8attn_varlen_fwd_sched")
    return out


def varlen_fwd_bf16(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, cu_seqlens,
                    max_seqlen: int, softmax_scale: float = 0.0,
                    out: Optional[torch.Tensor] = None, error: Optional[torch.Tensor] = None,
                    stream=None) -> torch.Tensor:
    """Native bf16 attention for skipped layers or steps (bf16 MMAs, P kept in
    TMEM, running row max, no quantisation)."""
    T, H, cu, out = _attn_common(q, k, v, cu_seqlens, out, torch.bfloat16)
    _check(lib().fp8attn_varlen_fwd_bf16(_ptr(q), _ptr(k), _ptr(v), _ptr(cu), cu.numel() - 1,
                                         int(max_seqlen), T, H, HEAD_DIM, float(softmax_scale),
                                         _ptr(out), _ptr(error),
                                         ctypes.c_void_p(_stream(stream, q.device))),
           "fp8attn_varlen_fwd_bf16")
    return out


def read_error_word(error: torch.Tensor, stream=None) -> int:
    """Read and clear an attention error word (int32 CUDA tensor)."""
    _require_cuda(error, "error")
    return int(lib().fp8attn_read_error_word(_ptr(error),
                                             ctypes.c_void_p(_stream(stream, error.device))))


# ---------------------------------------------------------------------------
# helpers
# ---------------------------------------------------------------------------

def parse_selector(text: Optional[str], max_index: int) -> set:
    """Indices selected by "0,1,4-6"-style selectors (via the C parser)."""
    mask = np.zeros(max(int(max_index), 1), dtype=np.uint8)
    raw = None if text is None else text.encode()
    _check(lib().fp8attn_parse_selector(raw, int(max_index), mask.ctypes.data_as(ctypes.c_void_p)),
           "fp8attn_parse_selector")
    return set(int(i) for i in np.nonzero(mask[:max_index])[0])


def e4m3_encode(x: torch.Tensor, scale: float = 1.0, stream=None) -> torch.Tensor:
    """E4M3 codes of fl32(x * scale) for an fp32 CUDA tensor (the kernel's cast)."""
    _require_cuda(x, "x")
    if x.dtype != torch.float32:
        raise ValueError("x must be float32")
    x = x.contiguous()
    out = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
    _check(lib().fp8attn_e4m3_encode(_ptr(x), x.numel(), float(scale), _ptr(out),
                                     ctypes.c_void_p(_stream(stream, x.device))),
           "fp8attn_e4m3_encode")
    return out


def quantize_qkv_noalloc(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, cu_seqlens,
                         max_seqlen: int, q8: torch.Tensor, k8: torch.Tensor, v8: torch.Tensor,
                         descale_out: torch.Tensor, scale_out: Optional[torch.Tensor] = None, *,
                         total_tokens: Optional[int] = None, src_seq_start=None,
                         stream=None) -> None:
    """Allocation-free one-shot dynamic quantisation (scales from this call's
    amax; no context, no workspace).  For callers that cannot allocate device
    memory: every buffer, including the outputs ``q8``/``k8``/``v8`` and the
    3-float ``descale_out`` (and optional ``scale_out``), is the caller's, and
    the library keeps its reduction scratch in a fixed device array.  Calls
    that overlap on the GPU race on that array.  Sources are checked as for
    :meth:`Context.quantize_qkv`; the call runs with ``q``'s device current
    (the library's array belongs to the current device)."""
    H, tok_stride, head_stride, cu, B, total_tokens, sss = _qkv_source(
        q, k, v, cu_seqlens, total_tokens, src_seq_start)
    if cu.device != q.device or (sss is not None and sss.device != q.device):
        raise ValueError(f"cu_seqlens and src_seq_start must be on {q.device}")
    for name, t in (("q8", q8), ("k8", k8), ("v8", v8)):
        _check_out(t, name, torch.uint8, int(total_tokens) * H * HEAD_DIM, q.device)
    _check_out(descale_out, "descale_out", torch.float32, 3, q.device)
    if scale_out is not None:
        _check_out(scale_out, "scale_out", torch.float32, 3, q.device)
    with torch.cuda.device(q.device):
        _check(lib().fp8attn_quantize_qkv_noalloc(
            _ptr(q), _ptr(k), _ptr(v), tok_stride, head_stride, _ptr(sss), _ptr(cu), B,
            int(max_seqlen), int(total_tokens), H, HEAD_DIM, _ptr(q8), _ptr(k8), _ptr(v8),
            _ptr(descale_out), _ptr(scale_out), ctypes.c_void_p(_stream(stream, q.device))),
            "fp8attn_quantize_qkv_noalloc")


def quantize_qkv_noalloc_error(stream=None) -> int:
    """Read and clear the allocation-free entry point's device error word."""
    return int(lib().fp8attn_quantize_qkv_noalloc_error(
        ctypes.c_void_p(_stream(stream, torch.cuda.current_device()))))


def launch_count() -> int:
    """Kernels launched by the library so far in this process."""
    return int(lib().fp8attn_launch_count())


SCALE_NAME_MAX = 256   # FP8ATTN_SCALE_NAME_MAX


def apply_margin(values, margin: float = DEFAULT_MARGIN) -> np.ndarray:
    """fl32(value * margin) for each value (fp8attn_apply_margin): the save
    margin of the vLLM FP8 ViT page, applied in the library."""
    v = np.ascontiguousarray(np.asarray(values, dtype=np.float32))
    out = np.empty_like(v)
    _check(lib().fp8attn_apply_margin(v.ctypes.data_as(ctypes.c_void_p), v.size,
                                      float(margin), out.ctypes.data_as(ctypes.c_void_p)),
           "fp8attn_apply_margin")
    return out


def load_scale_file(path: str, margin: float = 1.0) -> Dict[str, Tuple[float, float, float]]:
    """Read a per-layer {"q","k","v"} scale map (``q_scale``/``k_scale``/
    ``v_scale`` accepted as aliases), as in the vLLM FP8 ViT page's scale
    file format section, through fp8attn_scale_map_parse.

    The page applies its save margin when the file is written, so by default
    the values are used as stored (``margin=1.0``).  A file written without
    the margin can be read with it applied here: each value becomes
    fl32(value * margin) (in the library)."""
    with open(path, "rb") as f:
        text = f.read()
    cap = max(1, text.count(b":"))          # at least one ':' per layer
    names = ctypes.create_string_buffer(cap * SCALE_NAME_MAX)
    values = np.zeros((cap, 3), dtype=np.float32)
    n = ctypes.c_int(0)
    status = lib().fp8attn_scale_map_parse(text, len(text), float(margin), cap, names,
                                           values.ctypes.data_as(ctypes.c_void_p),
                                           ctypes.byref(n))
    if status != 0:
        raise ValueError(f"{path}: not a valid scale map (or margin {margin} not allowed)")
    out = {}
    for i in range(n.value):
        raw = names.raw[i * SCALE_NAME_MAX:(i + 1) * SCALE_NAME_MAX]
        out[raw[:raw.index(b"\0")].decode()] = tuple(float(x) for x in values[i])
    return out


def save_scale_file(path: str, layer_names: Sequence[str], values: np.ndarray) -> None:
    """Write exported values ([L, 3]) as a per-layer {"q","k","v"} map
    (fp8attn_scale_map_format)."""
    values = np.ascontiguousarray(np.asarray(values, dtype=np.float32).reshape(len(layer_names), 3))
    names = ctypes.create_string_buffer(max(1, len(layer_names)) * SCALE_NAME_MAX)
    for i, n in enumerate(layer_names):
        b = n.encode()
        if len(b) >= SCALE_NAME_MAX or b"\0" in b:
            raise ValueError(f"layer name {n!r} too long or holds a NUL")
        ctypes.memmove(ctypes.addressof(names) + i * SCALE_NAME_MAX, b, len(b))
    need = ctypes.c_size_t(0)
    L = lib()
    L.fp8attn_scale_map_format(len(layer_names), names, values.ctypes.data_as(ctypes.c_void_p),
                               None, 0, ctypes.byref(need))
    buf = ctypes.create_string_buffer(need.value)
    _check(L.fp8attn_scale_map_format(len(layer_names), names,
                                      values.ctypes.data_as(ctypes.c_void_p), buf, need.value,
                                      ctypes.byref(need)), "fp8attn_scale_map_format")
    with open(path, "wb") as f:
        f.write(buf.value)


def selftest_qk_scores(q8: torch.Tensor, k8: torch.Tensor, stream=None) -> torch.Tensor:
    """S = Q K^T for 128 x 128 tiles of E4M3 codes with the attention kernel's
    MMA sequence: q8, k8 uint8 [tiles * 128, 128] on the device; returns fp32
    [tiles, 128, 128] (a self-test of the tensor cores' accumulation)."""
    for name, t in (("q8", q8), ("k8", k8)):
        _require_cuda(t, name)
        if t.dtype != torch.uint8 or not t.is_contiguous() or t.dim() != 2 or \
                t.shape[1] != HEAD_DIM or t.shape[0] % 128 or t.shape[0] == 0:
            raise ValueError(f"{name} must be a contiguous uint8 [tiles * 128, 128] tensor")
    if q8.shape != k8.shape:
        raise ValueError("q8 and k8 must have the same shape")
    tiles = q8.shape[0] // 128
    out = torch.empty((tiles, 128, 128), dtype=torch.float32, device=q8.device)
    err = torch.zeros(1, dtype=torch.int32, device=q8.device)
    _check(lib().fp8attn_selftest_qk_scores(_ptr(q8), _ptr(k8), tiles, _ptr(out), _ptr(err),
                                            ctypes.c_void_p(_stream(stream, q8.device))),
           "fp8attn_selftest_qk_scores")
    _check(read_error_word(err, stream), "fp8attn_selftest_qk_scores (device)")
    return out


def selftest_bounded_waits(mbar_limit_ns: int = 50_000_000, device=None) -> int:
    """Run the library's two wait probes (an mbarrier wait and a grid barrier
    that nothing completes) and return how many gave up at their limit (2 when
    the bounds work).  Takes about one second."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    n = ctypes.c_int(-1)
    _check(lib().fp8attn_selftest_bounded_waits(int(mbar_limit_ns), ctypes.byref(n),
                                                ctypes.c_void_p(_stream(None, dev))),
           "fp8attn_selftest_bounded_waits")
    return n.value


def head_sharded_dynamic_quantize(ctx: "Context", layer: int, q: torch.Tensor, k: torch.Tensor,
                                  v: torch.Tensor, cu_seqlens, max_seqlen: int, group=None,
                                  out: Optional[Sequence[torch.Tensor]] = None, stream=None,
                                  comm=None) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """One dynamic pass over this rank's heads of a layer whose heads are
    sharded across the ranks of `group` (torch.distributed, NCCL on GPUs):
    local amax -> all-reduce MAX of the three values (the only exchange) ->
    push into this rank's ring -> cast this shard with the ring scales.  Every
    rank ends with the ring, scales and codes one DYNAMIC pass over all heads
    would give.  With no process group (or one rank) it is the same sequence
    without the all-reduce.  The exchange goes through ``comm`` (default: a
    :class:`TorchComm` over ``group``)."""
    comm = TorchComm(group) if comm is None else comm
    amax = ctx.amax_qkv(q, k, v, cu_seqlens, max_seqlen, stream=stream)
    if comm.size() > 1:
        cm = torch.cuda.stream(stream if isinstance(stream, torch.cuda.Stream)
                               else torch.cuda.ExternalStream(int(stream))) \
            if stream is not None else contextlib.nullcontext()
        with cm:
            comm.all_reduce_max(amax)
    ctx.amax_ring_update(layer, amax, stream=stream)
    return ctx.quantize_qkv(layer, RING, q, k, v, cu_seqlens, max_seqlen, out=out, stream=stream)


def regroup_heads(x: torch.Tensor, groups: int, to_groups: bool = True,
                  out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Head-group regrouping around the all-to-all of sequence-parallel
    attention: [T, H, 128] -> [groups, T, H/groups, 128] (``to_groups``) or
    back.  bf16 or uint8 (E4M3 codes), contiguous, on the device."""
    _require_cuda(x, "x")
    if x.dtype not in (torch.bfloat16, torch.uint8) or not x.is_contiguous():
        raise ValueError("x must be a contiguous bf16 or uint8 tensor")
    groups = int(groups)
    if to_groups:
        if x.dim() != 3 or x.shape[-1] != HEAD_DIM:
            raise ValueError("x must be [T, H, 128]")
        T, H, _ = x.shape
        if groups < 1 or H % groups:
            raise ValueError("num_heads must be a multiple of groups")
        shape = (groups, T, H // groups, HEAD_DIM)
    else:
        if x.dim() != 4 or x.shape[0] != groups or x.shape[-1] != HEAD_DIM:
            raise ValueError("x must be [groups, T, H/groups, 128]")
        _, T, Hn, _ = x.shape
        H = groups * Hn
        shape = (T, H, HEAD_DIM)
    if out is None:
        out = torch.empty(shape, dtype=x.dtype, device=x.device)
    elif tuple(out.shape) != shape or out.dtype != x.dtype or not out.is_contiguous():
        raise ValueError(f"out must be a contiguous {shape} {x.dtype} tensor")
    _check(lib().fp8attn_regroup_heads(_ptr(x), _ptr(out), T, H, groups,
                                       HEAD_DIM * x.element_size(), int(bool(to_groups)),
                                       ctypes.c_void_p(_stream(stream, x.device))),
           "fp8attn_regroup_heads")
    return out


class TorchComm:
    """The exchanges of the sharded paths over a torch.distributed process
    group (NCCL between GPUs).  Without an initialised process group it is a
    single rank and exchanges nothing."""

    def __init__(self, group=None):
        import torch.distributed as dist
        self._dist = dist
        self.group = group
        self._on = dist.is_available() and dist.is_initialized()

    def size(self) -> int:
        return self._dist.get_world_size(self.group) if self._on else 1

    def rank(self) -> int:
        return self._dist.get_rank(self.group) if self._on else 0

    def all_reduce_max(self, t: torch.Tensor) -> None:
        if self.size() > 1:
            self._dist.all_reduce(t, op=self._dist.ReduceOp.MAX, group=self.group)

    def all_to_all(self, out: torch.Tensor, inp: torch.Tensor) -> None:
        """Chunk i of ``inp`` (split along dim 0) goes to rank i; chunk i of
        ``out`` comes from rank i."""
        self._dist.all_to_all_single(out, inp, group=self.group)


_SINGLE_SEQ_CU: Dict[Tuple[str, int], torch.Tensor] = {}


def _single_seq_cu(S: int, device) -> torch.Tensor:
    """Device cu_seqlens [0, S], made once per (device, S): later calls copy
    nothing from the host, so they can be captured in a CUDA graph."""
    key = (str(torch.device(device)), int(S))
    t = _SINGLE_SEQ_CU.get(key)
    if t is None:
        t = _cu_tensor([0, int(S)], device)
        _SINGLE_SEQ_CU[key] = t
    return t


def ulysses_attention(ctx: "Context", layer: int, mode: int, q: torch.Tensor, k: torch.Tensor,
                      v: torch.Tensor, comm=None, softmax_scale: float = 0.0,
                      stream=None, p_rule: int = P_LINEAR_LOG,
                      schedule: int = SCHED_AUTO) -> torch.Tensor:
    """Sequence-parallel (Ulysses) attention over one sequence whose tokens are
    split evenly across the ranks of ``comm`` (a :class:`TorchComm` by
    default): rank r holds tokens [r S_loc, (r+1) S_loc) of Q, K, V as bf16
    [S_loc, H, 128]; it returns the same tokens of the output, bf16
    [S_loc, H, 128].  vLLM-Omni docs, "Quantized KV Cache", Configuration:
    the offline diffusion example shards the DiT over a Ulysses degree of 4.

    FP8 modes quantise BEFORE the exchange, so the all-to-all moves 1-byte
    codes: DYNAMIC takes the amax of this rank's tokens (all heads), the
    all-reduce MAX of the three values makes it the amax of the whole
    sequence, the ring is updated, and each group of H/n heads is cast with
    the ring scales straight into its send chunk; STATIC casts with the
    layer's static bounds.  Then: all-to-all (rank r receives every rank's
    tokens of head group r, i.e. the whole sequence in token order), attention
    on those heads, the return all-to-all, and the inverse head regrouping.
    SKIP regroups and exchanges bf16 and runs the bf16 attention.  Codes,
    scales, ring and output equal one single-GPU pass over the whole sequence
    (``quantize_qkv`` with the same mode, then ``varlen_fwd``), bit for bit
    under any work ``schedule``.  Every rank must make the same calls in the
    same order."""
    comm = TorchComm() if comm is None else comm
    n = int(comm.size())
    if q.dim() != 3 or q.shape != k.shape or q.shape != v.shape:
        raise ValueError("q, k, v must be [S_local, H, 128] of the same shape")
    if mode not in (DYNAMIC, STATIC, SKIP):
        raise ValueError("mode must be DYNAMIC, STATIC or SKIP")
    S_loc, H, D = q.shape
    if D != HEAD_DIM:
        raise ValueError("head_dim must be 128")
    if H % n:
        raise ValueError("num_heads must be a multiple of the number of ranks")
    Hn, S = H // n, S_loc * n
    dev = q.device
    cm = torch.cuda.stream(stream if isinstance(stream, torch.cuda.Stream)
                           else torch.cuda.ExternalStream(int(stream))) \
        if stream is not None else contextlib.nullcontext()
    with cm:
        cu_loc = _single_seq_cu(S_loc, dev)
        cu_all = _single_seq_cu(S, dev)
        if mode == SKIP:
            send = [regroup_heads(x.contiguous(), n) if n > 1 else x.contiguous()
                    for x in (q, k, v)]
        else:
            cast = STATIC
            if mode == DYNAMIC:
                amax = ctx.amax_qkv(q, k, v, cu_loc, S_loc)
                comm.all_reduce_max(amax)
                ctx.amax_ring_update(layer, amax)
                cast = RING
            # one launch casts every head group straight into its send chunk
            send = list(ctx.quantize_qkv_grouped(layer, cast, q, k, v, cu_loc, S_loc, n))
        if n > 1:
            recv = [torch.empty_like(x) for x in send]
            for r, x in zip(recv, send):
                comm.all_to_all(r, x)
        else:
            recv = send
        recv = [x.view(S, Hn, D) for x in recv]
        if mode == SKIP:
            o = varlen_fwd_bf16(recv[0], recv[1], recv[2], cu_all, S, softmax_scale)
        else:
            o = varlen_fwd(recv[0], recv[1], recv[2], cu_all, S, ctx.descale_ptr(layer),
                           softmax_scale, p_rule=p_rule, schedule=schedule)
        if n == 1:
            return o.view(S_loc, H, D)
        back = torch.empty_like(o)
        comm.all_to_all(back, o)
        return regroup_heads(back.view(n, S_loc, Hn, D), n, to_groups=False)
