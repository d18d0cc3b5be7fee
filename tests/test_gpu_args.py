"""Caller-provided output buffers are checked on the host before any launch:
a buffer that is too small, of another dtype or not contiguous raises, and
nothing is written."""
import pytest
import torch

import synthetic
import quantization_amax_reduce_b200 as qar

pytestmark = pytest.mark.gpu

DEV = "cuda"


def test_output_buffers_are_checked_before_launch():
    q, k, v, cu = synthetic.small_qkv(3, [100, 28], H=2, device=DEV)
    cu_d = torch.as_tensor(cu, device=DEV)
    ctx = qar.Context(1)
    n0 = qar.launch_count()
    small = [torch.zeros(127, 2, 128, dtype=torch.uint8, device=DEV) for _ in range(3)]
    with pytest.raises(ValueError, match="needed"):
        ctx.quantize_qkv(0, qar.DYNAMIC, q, k, v, cu_d, 100, out=small)
    wrong = [torch.zeros(128, 2, 128, dtype=torch.int8, device=DEV) for _ in range(3)]
    with pytest.raises(ValueError, match="contiguous"):
        ctx.quantize_qkv(0, qar.DYNAMIC, q, k, v, cu_d, 100, out=wrong)
    strided = [torch.zeros(128, 4, 128, dtype=torch.uint8, device=DEV)[:, :2] for _ in range(3)]
    with pytest.raises(ValueError, match="contiguous"):
        ctx.quantize_qkv(0, qar.DYNAMIC, q, k, v, cu_d, 100, out=strided)
    with pytest.raises(ValueError, match="three"):
        ctx.quantize_qkv(0, qar.DYNAMIC, q, k, v, cu_d, 100, out=small[:2])
    with pytest.raises(ValueError):
        ctx.amax_qkv(q, k, v, cu_d, 100, out=torch.zeros(3, dtype=torch.float64, device=DEV))
    with pytest.raises(ValueError, match="needed"):
        ctx.amax_qkv(q, k, v, cu_d, 100, out=torch.zeros(2, dtype=torch.float32, device=DEV))
    q8, k8, v8 = ctx.quantize_qkv(0, qar.DYNAMIC, q, k, v, cu_d, 100)
    n1 = qar.launch_count()
    out = torch.zeros(127, 2, 128, dtype=torch.bfloat16, device=DEV)
    with pytest.raises(ValueError, match="needed"):
        qar.varlen_fwd(q8, k8, v8, cu_d, 100, ctx.descale_ptr(0), out=out)
    with pytest.raises(ValueError, match="needed"):
        qar.varlen_fwd_bf16(q, k, v, cu_d, 100, out=out)
    ds = torch.zeros(3, dtype=torch.float32, device=DEV)
    with pytest.raises(ValueError, match="needed"):
        qar.quantize_qkv_noalloc(q, k, v, cu_d, 100, *small, ds)
    with pytest.raises(ValueError, match="source rows"):
        ctx.quantize_qkv(0, qar.DYNAMIC, q, k, v, cu_d, 100, total_tokens=129)
    # only the one good quantisation launched
    assert n1 == n0 + 1 and qar.launch_count() == n1


def test_noalloc_checks_and_counts_its_launch():
    """The allocation-free entry point refuses a total_tokens beyond the
    source rows before launching, and a good call counts as one launch."""
    q, k, v, cu = synthetic.small_qkv(4, [100, 28], H=2, device=DEV)
    cu_d = torch.as_tensor(cu, device=DEV)
    outs = [torch.zeros(129, 2, 128, dtype=torch.uint8, device=DEV) for _ in range(3)]
    ds = torch.zeros(3, dtype=torch.float32, device=DEV)
    n0 = qar.launch_count()
    with pytest.raises(ValueError, match="source rows"):
        qar.quantize_qkv_noalloc(q, k, v, cu_d, 100, *outs, ds, total_tokens=129)
    with pytest.raises(ValueError, match="CUDA tensor"):
        qar.quantize_qkv_noalloc(q, k, v, cu_d, 100, *outs, torch.zeros(3, dtype=torch.float32))
    assert qar.launch_count() == n0
    qar.quantize_qkv_noalloc(q, k, v, cu_d, 100, *outs, ds)
    torch.cuda.synchronize()
    assert qar.quantize_qkv_noalloc_error() == 0
    assert qar.launch_count() == n0 + 1
