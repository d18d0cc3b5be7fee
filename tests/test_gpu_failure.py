"""Failure detection on the GPU without a fault: waits that nothing completes
give up at their limit, report it, and leave the GPU usable.

Every wait inside the kernels (mbarrier waits in the attention kernels, the
grid barrier in the quantisation kernels) is bounded; the library's self-test
runs one probe of each whose condition is never met."""
import time

import numpy as np
import pytest
import torch

import oracle
import synthetic
import quantization_amax_reduce_b200 as qar
from tests.parity import assert_attention_close

pytestmark = pytest.mark.gpu

DEV = "cuda"


def test_waits_give_up_at_their_limit_and_the_gpu_stays_usable():
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    gave_up = qar.selftest_bounded_waits(50_000_000)      # 50 ms mbarrier limit
    dt = time.perf_counter() - t0
    assert gave_up == 2
    # the grid-barrier probe waits the library's full 1 s limit
    assert 1.0 <= dt < 10.0, dt
    # a normal quantise + attention pass afterwards still matches the oracle
    lens = [300, 17]
    q, k, v, cu = synthetic.small_qkv(41, lens, H=2, scale=1.0, device=DEV)
    cu_d = torch.as_tensor(cu, device=DEV)
    ctx = qar.Context(1)
    q8, k8, v8 = ctx.quantize_qkv(0, qar.DYNAMIC, q, k, v, cu_d, max(lens))
    out = qar.varlen_fwd(q8, k8, v8, cu_d, max(lens), ctx.descale_ptr(0))
    torch.cuda.synchronize()
    assert ctx.get_error() == 0
    qs, ds = ctx.get_scales(0)
    want = oracle.attention_fp8(q8.cpu().numpy(), k8.cpu().numpy(), v8.cpu().numpy(), cu,
                                [float(x) for x in ds], return_alternative=True)
    assert_attention_close(out, want, what="after the wait probes")
