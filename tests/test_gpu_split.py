"""GPU parity of the FP8 attention kernel's work schedules.

A work unit (256 query rows of one head of one sequence) is computed as two
128-row tiles.  It runs either in one CTA that interleaves both tiles or as
two CTAs of one tile each; the automatic schedule uses the second form for
the units of a mostly empty last wave, and for all units when they fit in a
single wave that fills at most half the SMs.  Every output row goes through the
same key blocks, in the same order, under the same P rule either way, so the
schedules must agree bit for bit, and each must match the oracle."""
import numpy as np
import pytest
import torch

import oracle
import quantization_amax_reduce_b200 as qar
from tests.parity import assert_attention_close, sample_rows

pytestmark = pytest.mark.gpu

DEV = "cuda"
RULES = [pytest.param(qar.P_LINEAR_LOG, oracle.P_LINEAR_LOG, id="linear_log"),
         pytest.param(qar.P_EXP2, oracle.P_EXP2, id="exp2")]
SCHEDULES = [(qar.SCHED_WHOLE, "whole"), (qar.SCHED_SPLIT, "split"), (qar.SCHED_AUTO, "auto")]


def _codes(T, H, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(T, H, 128, generator=g) * scale
    return x.to(torch.float8_e4m3fn).view(torch.uint8)


def _run(q8, k8, v8, cu, ds, rule, schedule, scale=0.0):
    return qar.varlen_fwd(q8.to(DEV), k8.to(DEV), v8.to(DEV), torch.as_tensor(cu, device=DEV),
                          int(np.max(np.diff(cu))), torch.as_tensor(ds, device=DEV),
                          softmax_scale=scale, p_rule=rule, schedule=schedule)


@pytest.mark.parametrize("rule,orule", RULES)
@pytest.mark.parametrize("lens,H", [
    ([5000, 300, 8269], 2),       # 198 units: AUTO splits the last 50 on 148 SMs
    ([129, 1, 257, 40], 3),       # 24 units: AUTO splits them all; empty second tiles
    ([1000, 17], 40),             # 200 units, ragged sequences
])
def test_schedules_agree_bit_for_bit_and_with_the_oracle(lens, H, rule, orule):
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    T = int(cu[-1])
    q8, k8, v8 = (_codes(T, H, s, 6.0) for s in (41, 42, 43))
    ds = [0.05, 0.04, 1.0 / 60.0]
    outs = {name: _run(q8, k8, v8, cu, ds, rule, sched) for sched, name in SCHEDULES}
    torch.cuda.synchronize()
    for name in ("split", "auto"):
        assert torch.equal(outs[name], outs["whole"]), f"{name} vs whole, {lens} H={H} {orule}"
    rows = sample_rows(cu, 48, seed=7)
    want = oracle.attention_fp8(q8.numpy(), k8.numpy(), v8.numpy(), cu, ds, rows=rows,
                                return_alternative=True, rule=orule)
    assert_attention_close(outs["split"], want, rows=rows,
                           what=f"schedules {lens} H={H}, split {orule}")


def _wide_range_case(start):
    """One head, 8192 keys, q = e_0 and softmax scale 1, so every row's
    scores are k[:, 0]: the first half around 0 with one key at 8; from key
    4096 the scores open at `start` and climb block by block to about 7."""
    n, D = 8192, 128
    g = torch.Generator().manual_seed(int(abs(start)) + 5)
    s = torch.randn(n, generator=g) * 0.5
    s[0] = 8.0
    blk = torch.arange(n) // 128
    ramp = start + (7.0 - start) * (blk - 32).clamp(min=0).float() / 31.0
    s = torch.where(blk >= 32, ramp + torch.randn(n, generator=g) * 0.25, s)
    q = torch.zeros(n, 1, D)
    q[:, 0, 0] = 1.0
    k = torch.zeros(n, 1, D)
    k[:, 0, 0] = s
    q8 = q.to(torch.float8_e4m3fn).view(torch.uint8)
    k8 = k.to(torch.float8_e4m3fn).view(torch.uint8)
    v8 = _codes(n, 1, 77, 4.0)
    return q8, k8, v8


@pytest.mark.parametrize("rule,orule", RULES)
@pytest.mark.parametrize("start", [-20.0, -200.0])
def test_scores_spanning_hundreds_of_log2_units(rule, orule, start):
    # keys far below the reference underflow to code 0, then the reference
    # moves up block by block as the scores climb back
    q8, k8, v8 = _wide_range_case(start)
    cu = np.array([0, q8.shape[0]], dtype=np.int32)
    ds = [1.0, 1.0, 1.0 / 8.0]
    rows = np.array([0, 1, 127, 128, 255, 4096, 8191], dtype=np.int64)
    want = oracle.attention_fp8(q8.numpy(), k8.numpy(), v8.numpy(), cu, ds, scale=1.0,
                                rows=rows, return_alternative=True, rule=orule)
    outs = {name: _run(q8, k8, v8, cu, ds, rule, sched, scale=1.0) for sched, name in SCHEDULES}
    torch.cuda.synchronize()
    assert torch.equal(outs["split"], outs["whole"])
    assert torch.isfinite(outs["whole"].float()).all()
    assert_attention_close(outs["whole"], want, rows=rows,
                           what=f"score range from {start}, {orule}")


def _split_sized_case(seed):
    # 512 units (S=8192, 16 heads): on 148 SMs the automatic schedule runs
    # the last 68 as single-tile CTAs in a second launch behind the first
    S, H = 8192, 16
    q8, k8, v8 = (_codes(S, H, seed + s, 6.0) for s in range(3))
    return [x.to(DEV) for x in (q8, k8, v8)], torch.tensor([0, S], dtype=torch.int32, device=DEV)


def test_split_call_in_a_cuda_graph_matches_eager():
    (q8, k8, v8), cu = _split_sized_case(90)
    ds = torch.tensor([0.05, 0.04, 1.0 / 60.0], device=DEV)
    eager = qar.varlen_fwd(q8, k8, v8, cu, 8192, ds)
    out = torch.empty_like(eager)
    stream = torch.cuda.Stream()
    stream.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(stream):
        qar.varlen_fwd(q8, k8, v8, cu, 8192, ds, out=out, stream=stream)   # warm-up
    torch.cuda.current_stream().wait_stream(stream)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    out.zero_()
    with torch.cuda.graph(g, stream=stream):
        qar.varlen_fwd(q8, k8, v8, cu, 8192, ds, out=out, stream=stream)
    for _ in range(3):
        out.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(out, eager)


def test_back_to_back_split_calls_keep_stream_order():
    # two calls into the same output on one stream: every row must hold the
    # second call's result (the first call's single-tile launch may not end
    # after the second call has written)
    (qa, ka, va), cu = _split_sized_case(91)
    (qb, kb, vb), _ = _split_sized_case(95)
    ds = torch.tensor([0.05, 0.04, 1.0 / 60.0], device=DEV)
    want = qar.varlen_fwd(qb, kb, vb, cu, 8192, ds)
    out = torch.empty_like(want)
    for _ in range(3):
        qar.varlen_fwd(qa, ka, va, cu, 8192, ds, out=out)
        qar.varlen_fwd(qb, kb, vb, cu, 8192, ds, out=out)
        torch.cuda.synchronize()
        assert torch.equal(out, want)
