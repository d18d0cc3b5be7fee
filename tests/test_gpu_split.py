"""GPU parity of the FP8 attention kernel's split schedule.

A work unit (256 query rows of one head) can run as a pair of CTAs in one
cluster that take the two sides of a 4096-key segment boundary and combine
their halves of the output through distributed shared memory.  The P rule
restarts its reference max at every segment (fp8attn.h, fp8attn_p_rule), so
the split and the whole-row schedules compute the same rule: both are
compared with the oracle, and with each other to within bf16 rounding.
The rows below also cross the two places where a restart moves the scale of
O and l down: a second segment starting 28 log2 units below the first (O is
scaled up by 2^28) and one starting ~290 log2 units below (its first blocks
are dropped until the reference climbs back within 2^64)."""
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


def _codes(T, H, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(T, H, 128, generator=g) * scale
    return x.to(torch.float8_e4m3fn).view(torch.uint8)


def _run(q8, k8, v8, cu, ds, rule, schedule, scale=0.0):
    return qar.varlen_fwd(q8.to(DEV), k8.to(DEV), v8.to(DEV), torch.as_tensor(cu, device=DEV),
                          int(np.max(np.diff(cu))), torch.as_tensor(ds, device=DEV),
                          softmax_scale=scale, p_rule=rule, schedule=schedule)


def _close_to_each_other(a, b, what):
    a = a.float().cpu().numpy().astype(np.float64)
    b = b.float().cpu().numpy().astype(np.float64)
    fin = np.isfinite(a) & np.isfinite(b)
    assert np.array_equal(np.isfinite(a), np.isfinite(b)), what
    # the same fp32 values up to rounding order, each rounded to bf16: at
    # most a couple of bf16 spacings apart
    tol = 2.0 ** -7 * np.maximum(np.abs(a), np.abs(b)) + 1e-6
    d = np.abs(a - b)[fin]
    assert np.all(d <= tol[fin]), f"{what}: split vs whole max diff {d.max():.3e}"


@pytest.mark.parametrize("rule,orule", RULES)
def test_split_and_whole_schedules_agree_with_the_oracle(rule, orule):
    # 5000 keys split 4096 | 904; 8269 keys split 4096 | 4173 with a ragged
    # last block; 300 keys cannot be split and run whole in the pair's first CTA
    lens = [5000, 300, 8269]
    H = 2
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    T = int(cu[-1])
    q8, k8, v8 = (_codes(T, H, s, 6.0) for s in (41, 42, 43))
    ds = [0.05, 0.04, 1.0 / 60.0]
    whole = _run(q8, k8, v8, cu, ds, rule, qar.SCHED_WHOLE)
    split = _run(q8, k8, v8, cu, ds, rule, qar.SCHED_SPLIT)
    auto = _run(q8, k8, v8, cu, ds, rule, qar.SCHED_AUTO)
    torch.cuda.synchronize()
    _close_to_each_other(split, whole, f"varlen {lens} {orule}")
    # 198 units: on 148 SMs AUTO runs the last 50 as pairs (a second launch)
    _close_to_each_other(auto, whole, f"varlen {lens} {orule}, auto")
    rows = sample_rows(cu, 48, seed=7)
    want = oracle.attention_fp8(q8.numpy(), k8.numpy(), v8.numpy(), cu, ds, rows=rows,
                                return_alternative=True, rule=orule)
    assert_attention_close(whole, want, rows=rows, what=f"split test, whole {orule}")
    assert_attention_close(split, want, rows=rows, what=f"split test, split {orule}")


def _segment_drop_case(start):
    """One head, 8192 keys, q = e_0 and softmax scale 1, so every row's
    scores are k[:, 0]: the first segment around 0 with one key at 8; the
    second segment opens at `start` (block 32) and climbs block by block to
    about 7 at block 63."""
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
@pytest.mark.parametrize("start", [-20.0, -200.0], ids=["restart_scales_up", "restart_dropped"])
def test_segment_restart_far_below_the_first_segment(rule, orule, start):
    q8, k8, v8 = _segment_drop_case(start)
    cu = np.array([0, q8.shape[0]], dtype=np.int32)
    ds = [1.0, 1.0, 1.0 / 8.0]
    rows = np.array([0, 1, 255, 256, 4095, 4096, 8191], dtype=np.int64)
    want = oracle.attention_fp8(q8.numpy(), k8.numpy(), v8.numpy(), cu, ds, scale=1.0,
                                rows=rows, return_alternative=True, rule=orule)
    for sched, name in ((qar.SCHED_WHOLE, "whole"), (qar.SCHED_SPLIT, "split")):
        out = _run(q8, k8, v8, cu, ds, rule, sched, scale=1.0)
        torch.cuda.synchronize()
        assert torch.isfinite(out.float()).all()
        assert_attention_close(out, want, rows=rows,
                               what=f"segment restart from {start}, {name} {orule}")
