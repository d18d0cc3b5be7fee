"""GPU: the head-grouped cast (fp8attn_quantize_qkv_grouped) writes the same
codes as the packed cast, regrouped to [groups, T, H/groups, 128] -- the send
buffers of the sequence-parallel all-to-all (vLLM-Omni "Quantized KV Cache",
Configuration: the DiT sharded over a Ulysses degree).  Bit-exact for the
static and the ring-scale casts, packed and padded sources."""
import numpy as np
import pytest
import torch

import synthetic
import quantization_amax_reduce_b200 as qar

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _regroup(codes, groups):
    T, H, D = codes.shape
    return codes.view(T, groups, H // groups, D).permute(1, 0, 2, 3).contiguous()


@pytest.mark.parametrize("groups", [1, 2, 4, 8])
@pytest.mark.parametrize("mode", ["static", "ring"])
def test_grouped_cast_equals_packed_cast_regrouped(groups, mode):
    lens = [1000, 37, 4095]
    H = 16
    q, k, v, cu = synthetic.small_qkv(311, lens, H=H, scale=2.0, device=DEV)
    cu_d = torch.as_tensor(cu, device=DEV)
    ctx = qar.Context(1)
    if mode == "static":
        ctx.set_static_scales(0, 6.0, 5.5, 7.25)
        cast = qar.STATIC
    else:
        amax = ctx.amax_qkv(q, k, v, cu_d, max(lens))
        ctx.amax_ring_update(0, amax)
        cast = qar.RING
    packed = ctx.quantize_qkv(0, cast, q, k, v, cu_d, max(lens))
    grouped = ctx.quantize_qkv_grouped(0, cast, q, k, v, cu_d, max(lens), groups)
    torch.cuda.synchronize()
    assert ctx.get_error() == 0
    for a, b in zip(packed, grouped):
        assert b.shape == (groups, a.shape[0], H // groups, 128)
        assert torch.equal(b, _regroup(a, groups))


def test_grouped_cast_from_a_padded_source():
    lens, S_max, H, groups = [300, 129], 384, 8, 4
    q, k, v, cu = synthetic.small_qkv(312, lens, H=H, device=DEV)
    pads = []
    for x in (q, k, v):
        p = torch.full((len(lens), S_max, H, 128), float("nan"), dtype=torch.bfloat16, device=DEV)
        for b in range(len(lens)):
            p[b, :lens[b]] = x[cu[b]:cu[b + 1]]
        pads.append(p)
    starts = np.array([b * S_max for b in range(len(lens))], dtype=np.int32)
    ctx = qar.Context(1)
    ctx.set_static_scales(0, 4.0, 4.5, 5.0)
    cu_d = torch.as_tensor(cu, device=DEV)
    packed = ctx.quantize_qkv(0, qar.STATIC, q, k, v, cu_d, S_max)
    grouped = ctx.quantize_qkv_grouped(0, qar.STATIC, *pads, cu_d, S_max, groups,
                                       total_tokens=int(cu[-1]), src_seq_start=starts)
    torch.cuda.synchronize()
    for a, b in zip(packed, grouped):
        assert torch.equal(b, _regroup(a, groups))
