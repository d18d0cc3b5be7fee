"""A stand-in for ``quantization_amax_reduce_b200.Context`` whose every step
is the oracle's (CPU, test infrastructure): it lets multi-rank tests run the
product's host-side orchestration (the sharded and sequence-parallel helpers,
with their real torch.distributed exchanges over gloo) on CPU tensors.

vLLM docs, "FP8 ViT encoder attention", usage: a 16-entry ring of observed
amax values drives the per-tensor scales; static bounds come from a scale
file."""
import numpy as np
import torch

import oracle
import synthetic

D = 128


class OracleContext:
    """One layer's ring and scales, with the oracle doing each step."""

    def __init__(self, static_values=None):
        self.rings = [oracle.Ring() for _ in range(3)]
        self.qs = [np.float32(1.0)] * 3
        self.ds = [np.float32(1.0)] * 3
        self.static = static_values

    def amax_qkv(self, q, k, v, cu_seqlens, max_seqlen, *, total_tokens=None,
                 src_seq_start=None, out=None, stream=None):
        cu = np.asarray(cu_seqlens, dtype=np.int32)
        vals = []
        for x in (q, k, v):
            a, nf = oracle.amax(synthetic.bf16_bits(x.contiguous()), cu, x.shape[1], D)
            vals.append(float("inf") if nf else float(a))
        return torch.tensor(vals, dtype=torch.float32)

    def amax_ring_update(self, layer, amax3, stream=None):
        for t in range(3):
            a = float(amax3[t])
            bad = not np.isfinite(a)
            self.qs[t], self.ds[t] = self.rings[t].dynamic_step(0.0 if bad else a, bad)

    def quantize_qkv(self, layer, mode, q, k, v, cu_seqlens, max_seqlen, *, total_tokens=None,
                     src_seq_start=None, out=None, stream=None):
        from quantization_amax_reduce_b200 import RING, STATIC
        cu = np.asarray(cu_seqlens, dtype=np.int32)
        if mode == STATIC:
            sc = [oracle.scales_from_bound(np.float32(a)) for a in self.static]
            self.qs = [s[0] for s in sc]
            self.ds = [s[1] for s in sc]
        elif mode != RING:
            raise ValueError("the stand-in casts with RING or STATIC scales only")
        res = []
        for t, x in enumerate((q, k, v)):
            codes = torch.from_numpy(oracle.quantize(synthetic.bf16_bits(x.contiguous()), cu,
                                                     x.shape[1], D, self.qs[t]))
            if out is not None:
                out[t].copy_(codes)
                codes = out[t]
            res.append(codes)
        return tuple(res)

    def quantize_qkv_grouped(self, layer, mode, q, k, v, cu_seqlens, max_seqlen, groups, *,
                             total_tokens=None, src_seq_start=None, out=None, stream=None):
        codes = self.quantize_qkv(layer, mode, q, k, v, cu_seqlens, max_seqlen,
                                  total_tokens=total_tokens, src_seq_start=src_seq_start)
        res = []
        for t, c in enumerate(codes):
            T, Hh, Dd = c.shape
            g = c.view(T, groups, Hh // groups, Dd).permute(1, 0, 2, 3).contiguous()
            if out is not None:
                out[t].copy_(g)
                g = out[t]
            res.append(g)
        return tuple(res)

    def descale_ptr(self, layer):
        return [float(d) for d in self.ds]
