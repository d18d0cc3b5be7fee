"""Sequence-parallel (Ulysses) attention through the C ABI on one GPU.

The head regrouping kernel is checked against torch's permute.  For the whole
path, n ranks are emulated by n threads, each with its own context, whose
exchanges go through a thread-barrier stand-in for the process group (the
kernels of different ranks never wait on one another, so nothing here needs
the ranks to run at the same time).  Every rank's output, ring and scales must
equal one single-GPU pass over the whole sequence, bit for bit.

vLLM-Omni docs, "Quantized KV Cache", Configuration: the offline diffusion
example shards the DiT over a Ulysses degree of 4."""
import threading

import numpy as np
import pytest
import torch

import synthetic
import quantization_amax_reduce_b200 as qar

pytestmark = pytest.mark.gpu

DEV = "cuda"
STATIC_VALUES = (6.0, 5.5, 7.25)


# ---------------------------------------------------------------- regrouping

@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.uint8])
@pytest.mark.parametrize("T,H,G", [(1000, 8, 2), (1000, 8, 4), (1000, 8, 8), (1, 4, 2),
                                   (333, 40, 8), (77, 16, 1)])
def test_regroup_matches_permute_and_round_trips(dtype, T, H, G):
    g = torch.Generator(device=DEV).manual_seed(T * 100 + H * 10 + G)
    x = torch.randint(0, 256, (T, H, 128), generator=g, device=DEV, dtype=torch.int32)
    x = x.to(torch.uint8) if dtype == torch.uint8 else x.to(torch.bfloat16)
    y = qar.regroup_heads(x, G)
    want = x.view(T, G, H // G, 128).permute(1, 0, 2, 3).contiguous()
    assert y.shape == want.shape and torch.equal(y, want)
    z = qar.regroup_heads(y, G, to_groups=False)
    assert z.shape == x.shape and torch.equal(z, x)


def test_regroup_full_size_dit_slice():
    """One rank's slice of the 32760-token, 40-head sequence at degree 8."""
    g = torch.Generator(device=DEV).manual_seed(5)
    x = torch.randn(4095, 40, 128, generator=g, device=DEV).to(torch.bfloat16)
    y = qar.regroup_heads(x, 8)
    assert torch.equal(y, x.view(4095, 8, 5, 128).permute(1, 0, 2, 3))
    assert torch.equal(qar.regroup_heads(y, 8, to_groups=False), x)


def test_regroup_zero_tokens():
    x = torch.empty(0, 8, 128, dtype=torch.bfloat16, device=DEV)
    assert qar.regroup_heads(x, 4).shape == (4, 0, 2, 128)


# ---------------------------------------------------------- emulated ranks

class _Shared:
    def __init__(self, n):
        self.slots = [None] * n
        self.barrier = threading.Barrier(n, timeout=120)


class ThreadComm:
    """Rank `rank` of `n` threads; the exchanges copy between the ranks'
    device tensors after a barrier."""

    def __init__(self, rank, n, shared):
        self._rank, self._n, self._sh = rank, n, shared

    def size(self):
        return self._n

    def rank(self):
        return self._rank

    def _post(self, t):
        torch.cuda.synchronize()
        self._sh.slots[self._rank] = t
        self._sh.barrier.wait()
        return list(self._sh.slots)

    def _done(self):
        torch.cuda.synchronize()
        self._sh.barrier.wait()

    def all_reduce_max(self, t):
        parts = self._post(t.clone())
        r = parts[0].clone()
        for x in parts[1:]:
            r = torch.maximum(r, x)
        self._done()
        t.copy_(r)

    def all_to_all(self, out, inp):
        parts = self._post(inp)
        for i, x in enumerate(parts):
            out.view(self._n, -1)[i].copy_(x.view(self._n, -1)[self._rank])
        self._done()


def _run_ranks(n, fn):
    shared = _Shared(n)
    res, errs = [None] * n, []

    def body(r):
        try:
            res[r] = fn(r, ThreadComm(r, n, shared))
        except BaseException as e:   # noqa: BLE001 - reported below
            errs.append(e)
            shared.barrier.abort()

    th = [threading.Thread(target=body, args=(r,)) for r in range(n)]
    for t in th:
        t.start()
    for t in th:
        t.join(timeout=600)
    torch.cuda.synchronize()
    if errs:
        raise errs[0]
    assert all(not t.is_alive() for t in th)
    return res


def _single_pass(ctx, mode, q, k, v, S):
    cu = torch.tensor([0, S], dtype=torch.int32, device=DEV)
    if mode == qar.SKIP:
        return qar.varlen_fwd_bf16(q, k, v, cu, S)
    q8, k8, v8 = ctx.quantize_qkv(0, mode, q, k, v, cu, S)
    return qar.varlen_fwd(q8, k8, v8, cu, S, ctx.descale_ptr(0))


@pytest.mark.parametrize("n", [2, 4])
def test_emulated_ranks_equal_one_pass(n):
    H, S = 8, 1200
    S_loc = S // n
    plan = [qar.DYNAMIC, qar.DYNAMIC, qar.STATIC, qar.SKIP, qar.DYNAMIC, qar.DYNAMIC]
    full = qar.Context(1)
    ranks = [qar.Context(1) for _ in range(n)]
    for c in [full] + ranks:
        c.set_static_scales(0, *STATIC_VALUES)
    for p, mode in enumerate(plan):
        q, k, v, _ = synthetic.small_qkv(700 + p, [S], H=H, scale=1.0 + 0.5 * p, device=DEV)
        q[:, H - 1, 11] *= 8.0                  # head groups see different amax
        if p == 4:
            v[S - 3, 2, 64] = float("inf")      # non-finite amax: reported, not pushed
        want = _single_pass(full, mode, q, k, v, S)

        def fn(r, comm):
            mine = slice(r * S_loc, (r + 1) * S_loc)
            return qar.ulysses_attention(ranks[r], 0, mode, q[mine], k[mine], v[mine], comm=comm)

        got = _run_ranks(n, fn)
        for r in range(n):
            assert got[r].shape == (S_loc, H, 128)
            assert torch.equal(got[r], want[r * S_loc:(r + 1) * S_loc]), (p, mode, r)
        ws, wm = full.get_ring_state(0)
        for r in range(n):
            gs, gm = ranks[r].get_ring_state(0)
            np.testing.assert_array_equal(gs, ws)
            np.testing.assert_array_equal(gm, wm)
            for a, b in zip(ranks[r].get_scales(0), full.get_scales(0)):
                np.testing.assert_array_equal(a, b)
        e_full = full.get_error()
        assert (e_full != 0) == (p == 4), (p, e_full)
        assert all((c.get_error() != 0) == (p == 4) for c in ranks), p


def test_single_rank_without_a_process_group():
    H, S = 4, 500
    q, k, v, _ = synthetic.small_qkv(71, [S], H=H, scale=2.0, device=DEV)
    a, b = qar.Context(1), qar.Context(1)
    for mode in (qar.DYNAMIC, qar.SKIP):
        want = _single_pass(a, mode, q, k, v, S)
        got = qar.ulysses_attention(b, 0, mode, q, k, v)
        assert torch.equal(got, want), mode


def test_full_size_dit_sequence_at_degree_8():
    """The 32760-token, 40-head sequence split over 8 emulated ranks."""
    n = 8
    q, k, v, cu = synthetic.qkv(4, device=DEV)
    S, H = q.shape[0], q.shape[1]
    S_loc = S // n
    full = qar.Context(1)
    want = _single_pass(full, qar.DYNAMIC, q, k, v, S)
    ranks = [qar.Context(1) for _ in range(n)]

    def fn(r, comm):
        mine = slice(r * S_loc, (r + 1) * S_loc)
        return qar.ulysses_attention(ranks[r], 0, qar.DYNAMIC, q[mine], k[mine], v[mine],
                                     comm=comm)

    got = _run_ranks(n, fn)
    for r in range(n):
        assert torch.equal(got[r], want[r * S_loc:(r + 1) * S_loc]), r
    for r in range(n):
        for a, b in zip(ranks[r].get_scales(0), full.get_scales(0)):
            np.testing.assert_array_equal(a, b)
