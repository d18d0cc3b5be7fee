"""The allocation-free quantisation entry point against the context-based one.

fp8attn_quantize_qkv_noalloc serves callers that cannot allocate device
memory (an operator handed only its input and output buffers under a fixed
memory plan, or code that must not call cudaMalloc because it synchronises
the device): it keeps its reduction scratch in a fixed array inside the
library instead of a caller-provided workspace.  Its result must equal the
first dynamic pass of a fresh context, call after call, with the scratch
left over from the previous call (a larger launch with a larger amax)
having no effect on the next one.

This file sorts last so that a run stopping at the first failure has run
every other test before it.
"""
import numpy as np
import pytest
import torch

import synthetic
import quantization_amax_reduce_b200 as qar

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _context_pass(q, k, v, cu_d, max_len):
    ctx = qar.Context(1)
    q8, k8, v8 = ctx.quantize_qkv(0, qar.DYNAMIC, q, k, v, cu_d, max_len)
    qs, ds = ctx.get_scales(0)
    assert ctx.get_error() == 0
    return (q8, k8, v8), qs, ds


def _noalloc_pass(q, k, v, cu_d, max_len):
    T, H = q.shape[0], q.shape[1]
    outs = [torch.full((T, H, 128), 0xEE, dtype=torch.uint8, device=DEV) for _ in range(3)]
    descale = torch.full((3,), -1.0, dtype=torch.float32, device=DEV)
    scale = torch.full((3,), -1.0, dtype=torch.float32, device=DEV)
    qar.quantize_qkv_noalloc(q, k, v, cu_d, max_len, outs[0], outs[1], outs[2], descale, scale)
    torch.cuda.synchronize()
    assert qar.quantize_qkv_noalloc_error() == 0
    return outs, scale.cpu().numpy(), descale.cpu().numpy()


def test_noalloc_matches_context_path_on_two_calls_in_a_row():
    # call 1: a large varlen batch with a large amax (many CTAs);
    # call 2: a small input with a smaller amax (few CTAs)
    lens1 = [3000, 129, 5000]
    lens2 = [300, 17]
    q1, k1, v1, cu1 = synthetic.small_qkv(71, lens1, H=16, scale=5.0, device=DEV)
    q2, k2, v2, cu2 = synthetic.small_qkv(72, lens2, H=2, scale=1.0, device=DEV)
    for (q, k, v, cu, lens) in ((q1, k1, v1, cu1, lens1), (q2, k2, v2, cu2, lens2)):
        cu_d = torch.as_tensor(cu, device=DEV)
        want_codes, want_qs, want_ds = _context_pass(q, k, v, cu_d, max(lens))
        got_codes, got_qs, got_ds = _noalloc_pass(q, k, v, cu_d, max(lens))
        for g, w, name in zip(got_codes, want_codes, "qkv"):
            assert torch.equal(g, w), name
        np.testing.assert_array_equal(got_qs, want_qs)
        np.testing.assert_array_equal(got_ds, want_ds)
