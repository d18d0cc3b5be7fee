"""Seeded synthetic Q/K/V inputs shaped like the pages' attention workloads.

This module only draws random numbers; it holds none of the quantisation or
attention arithmetic.  Both the CUDA library's tests/benchmark and the CPU
oracle's tests take their inputs from here.

Workloads (the pages measure ViT-encoder and DiT attention with head_dim 128
at sequence lengths up to 8192 and beyond; no dataset is used -- these
synthetic draws stand in for image/video token activations):

* ``1``: one sequence, S=256, 2 heads, N(0,1)                 (dynamic, 1 pass)
* ``2``: 3 packed sequences, S_b ~ U{1024..8192}, 16 heads, N(0,1) with 1% of
  the (head, dim) channels scaled x20 as amax outliers      (dynamic, 16 passes)
* ``3``: one sequence, S=8192, 16 heads, N(0,1)              (static 224/198/210)
* ``4``: one sequence, S=32760, 40 heads; Q, K = N(0,1) + 3 U B with a shared
  per-token U in R^{S x 8} ~ N(0,1) and B ~ N(0, 1/8) per tensor; V = N(0,1)
                                                           (dynamic, 1 pass)
* ``5``: 24 layers x (4 sequences, S_b ~ U{4096..16384} per layer, 16 heads,
  Laplace(0,1)); 16 dynamic passes, export x1.5, static serve; layers 0-2 skip

Every tensor is drawn from a torch generator seeded with a SplitMix64 mix of
(config, layer, pass, tensor); sequence lengths and outlier channels come
from numpy's PCG64 seeded the same way.  Values are drawn in fp32 and rounded
to bf16 (round-to-nearest-even).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import List, Optional, Sequence, Tuple

import numpy as np
import torch

HEAD_DIM = 128
_MASK64 = (1 << 64) - 1


def splitmix64(x: int) -> int:
    """One SplitMix64 output step (Steele, Lea & Flood, 2014)."""
    x = (x + 0x9E3779B97F4A7C15) & _MASK64
    z = x
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _MASK64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _MASK64
    return z ^ (z >> 31)


def seed_for(*parts: int, base: int = 0) -> int:
    s = base
    for p in parts:
        s = splitmix64(s ^ (int(p) & _MASK64))
    return s & ((1 << 63) - 1)


_TENSOR_ID = {"q": 1, "k": 2, "v": 3, "u": 4, "lens": 5, "outq": 6, "outk": 7, "outv": 8,
              "bq": 9, "bk": 10}


@dataclass
class Workload:
    cid: int
    name: str
    B: int
    H: int
    lens: Optional[Tuple[int, ...]] = None          # fixed lengths
    len_range: Optional[Tuple[int, int]] = None     # inclusive uniform range
    dist: str = "normal"
    scaling: str = "dynamic"                        # dynamic | static
    passes: int = 1
    layers: int = 1
    static_values: Optional[Tuple[float, float, float]] = None
    skip_layers: str = ""
    D: int = HEAD_DIM

    def seq_lens(self, layer: int = 0) -> List[int]:
        if self.lens is not None:
            return list(self.lens)
        lo, hi = self.len_range
        rng = np.random.Generator(np.random.PCG64(seed_for(self.cid, layer, _TENSOR_ID["lens"])))
        return [int(v) for v in rng.integers(lo, hi + 1, size=self.B)]

    def cu_seqlens(self, layer: int = 0) -> np.ndarray:
        return np.concatenate([[0], np.cumsum(self.seq_lens(layer))]).astype(np.int32)

    def flops(self, layer: int = 0) -> float:
        """Algorithmic attention FLOPs: sum_b 4 S_b^2 D H."""
        return float(sum(4.0 * s * s * self.D * self.H for s in self.seq_lens(layer)))


WORKLOADS = {
    1: Workload(1, "single_seq_s256_h2", B=1, H=2, lens=(256,), dist="normal"),
    2: Workload(2, "vit_varlen3_s1024to8192_h16_outliers", B=3, H=16, len_range=(1024, 8192),
                dist="normal_outliers", passes=16),
    3: Workload(3, "kernel_s8192_h16_static", B=1, H=16, lens=(8192,), dist="normal",
                scaling="static", static_values=(224.0, 198.0, 210.0)),
    4: Workload(4, "dit_s32760_h40_lowrank", B=1, H=40, lens=(32760,), dist="lowrank"),
    5: Workload(5, "calibrate_serve_24l_varlen4_s4096to16384_h16_laplace", B=4, H=16,
                len_range=(4096, 16384), dist="laplace", passes=16, layers=24,
                skip_layers="0-2"),
}


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _normal(T: int, C: int, device, seed: int) -> torch.Tensor:
    return torch.randn(T, C, generator=_gen(device, seed), device=device, dtype=torch.float32)


def _laplace(T: int, C: int, device, seed: int) -> torch.Tensor:
    # inverse CDF of Laplace(0, 1): x = -sgn(w) ln(1 - 2|w|), w = u - 1/2
    u = torch.rand(T, C, generator=_gen(device, seed), device=device, dtype=torch.float32)
    w = u - 0.5
    a = (2.0 * w.abs()).clamp_(max=1.0 - 2.0 ** -24)
    return -torch.sign(w) * torch.log1p(-a)


def qkv(cid: int, layer: int = 0, pass_idx: int = 0, device="cpu"
        ) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor, np.ndarray]:
    """Packed bf16 (q, k, v) of shape [T, H, D] and cu_seqlens (int32)."""
    w = WORKLOADS[cid]
    cu = w.cu_seqlens(layer)
    T, H, D = int(cu[-1]), w.H, w.D
    C = H * D
    out = []
    if w.dist == "lowrank":
        U = _normal(T, 8, device, seed_for(cid, layer, pass_idx, _TENSOR_ID["u"]))
    for name in ("q", "k", "v"):
        s = seed_for(cid, layer, pass_idx, _TENSOR_ID[name])
        if w.dist == "laplace":
            x = _laplace(T, C, device, s)
        else:
            x = _normal(T, C, device, s)
        if w.dist == "normal_outliers":
            rng = np.random.Generator(np.random.PCG64(
                seed_for(cid, layer, pass_idx, _TENSOR_ID["out" + name])))
            n_out = C // 100   # 1% of the (head, dim) channels
            ch = torch.as_tensor(rng.choice(C, size=n_out, replace=False), device=device)
            x[:, ch] *= 20.0
        if w.dist == "lowrank" and name in ("q", "k"):
            Bm = _normal(8, C, device, seed_for(cid, layer, pass_idx, _TENSOR_ID["b" + name]))
            Bm *= 1.0 / math.sqrt(8.0)
            x += 3.0 * (U @ Bm)
        out.append(x.to(torch.bfloat16).view(T, H, D))
    return out[0], out[1], out[2], cu


def small_qkv(seed: int, lens: Sequence[int], H: int, D: int = HEAD_DIM,
              scale: float = 1.0, device="cpu"):
    """Small seeded N(0, scale^2) draws for unit tests of arbitrary shapes."""
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    T = int(cu[-1])
    res = []
    for i in range(3):
        x = _normal(T, H * D, device, seed_for(0xABC, seed, i)) * scale
        res.append(x.to(torch.bfloat16).view(T, H, D))
    return res[0], res[1], res[2], cu


def bf16_bits(x: torch.Tensor) -> np.ndarray:
    """Raw bf16 bit patterns of a CPU/GPU tensor as numpy uint16."""
    return x.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)
