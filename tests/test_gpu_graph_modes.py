"""A denoising loop with one captured CUDA graph per attention mode.

vLLM-Omni docs, parameters table: kv_cache_skip_steps lists denoising steps
that keep the native dtype; every other step runs the FP8 path (dynamic
scales from the device-resident amax ring).  Because the ring lives on the
device, the FP8 step (quantise + attention) is captured once and replayed;
the skipped steps replay a bf16 attention graph.  The replayed loop must give
the same ring state and bit-identical outputs as the same loop run eagerly.
"""
import numpy as np
import pytest
import torch

import oracle
import synthetic
import quantization_amax_reduce_b200 as qar

pytestmark = pytest.mark.gpu

DEV = "cuda"


def test_step_loop_replays_one_graph_per_mode():
    lens = [700, 333]
    H = 4
    n_steps = 8
    skip_steps = qar.parse_selector("0,5", n_steps)
    step_mask = np.zeros(n_steps, np.uint8)
    step_mask[sorted(skip_steps)] = 1
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    cu_d = torch.as_tensor(cu, device=DEV)
    T = int(cu[-1])
    inputs = [synthetic.small_qkv(300 + s, lens, H=H, scale=1.0 + 0.3 * s, device=DEV)[:3]
              for s in range(n_steps)]

    # eager reference loop
    eager = qar.Context(1)
    want = []
    for s, (q, k, v) in enumerate(inputs):
        mode = eager.select_mode_at_step(0, s, None, step_mask)
        assert mode == oracle.step_layer_mode(0, s, set(), skip_steps, False)
        if mode == qar.SKIP:
            want.append(qar.varlen_fwd_bf16(q, k, v, cu_d, max(lens)))
        else:
            q8, k8, v8 = eager.quantize_qkv(0, qar.DYNAMIC, q, k, v, cu_d, max(lens))
            want.append(qar.varlen_fwd(q8, k8, v8, cu_d, max(lens), eager.descale_ptr(0)))
    torch.cuda.synchronize()
    assert eager.get_error() == 0

    # one graph per mode over static buffers
    ctx = qar.Context(1)
    src = [torch.empty_like(inputs[0][i]) for i in range(3)]
    codes = [torch.empty((T, H, 128), dtype=torch.uint8, device=DEV) for _ in range(3)]
    out_fp8 = torch.empty((T, H, 128), dtype=torch.bfloat16, device=DEV)
    out_bf16 = torch.empty((T, H, 128), dtype=torch.bfloat16, device=DEV)
    stream = torch.cuda.Stream()
    stream.wait_stream(torch.cuda.current_stream())
    g_fp8, g_bf16 = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        with torch.cuda.graph(g_fp8, stream=stream):
            ctx.quantize_qkv(0, qar.DYNAMIC, src[0], src[1], src[2], cu_d, max(lens), out=codes,
                             stream=stream)
            qar.varlen_fwd(codes[0], codes[1], codes[2], cu_d, max(lens), ctx.descale_ptr(0),
                           out=out_fp8, stream=stream)
        with torch.cuda.graph(g_bf16, stream=stream):
            qar.varlen_fwd_bf16(src[0], src[1], src[2], cu_d, max(lens), out=out_bf16,
                                stream=stream)
    torch.cuda.current_stream().wait_stream(stream)
    for s, (q, k, v) in enumerate(inputs):
        for d, x in zip(src, (q, k, v)):
            d.copy_(x)
        if ctx.select_mode_at_step(0, s, None, step_mask) == qar.SKIP:
            g_bf16.replay()
            got = out_bf16
        else:
            g_fp8.replay()
            got = out_fp8
        torch.cuda.synchronize()
        assert torch.equal(got, want[s]), f"step {s}"
    assert ctx.get_error() == 0
    a_slots, a_meta = eager.get_ring_state(0)
    b_slots, b_meta = ctx.get_ring_state(0)
    np.testing.assert_array_equal(a_slots, b_slots)
    np.testing.assert_array_equal(a_meta, b_meta)
    # six FP8 steps pushed one amax each into every tensor's ring
    assert set(a_meta.reshape(-1).tolist()) == {n_steps - len(skip_steps)}
