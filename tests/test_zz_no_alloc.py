"""fa_bwd_noalloc: the backward for callers that cannot allocate device memory
(a host application that owns all device memory and hands out only input and
output buffers, or code that must not call cudaMalloc). It takes no
workspace and uses the library's built-in 64 MiB device scratch instead.

Its results must match the workspace entry point fa_bwd on the same inputs
(the same kernels: dK and dV bit-identical, dQ within the spread of its
atomic summation order), on two calls in a row: the second call reuses the
scratch the first one left behind. One call is also held to the oracle at
the parity tolerance the other tests use.
This file is collected last so that a run that stops at the first failure has
already run every other test.
"""
import pytest
import torch

import oracle
from exact_io_aware_96_b200 import fa
from exact_io_aware_96_b200.inputs import random_case
from tests.parity import check_grad, np64, rel_l2

A = 0x10000  # aligned placeholder address for host-side argument checks


def _ptr(t):
    return t.data_ptr()


def _bwd_both(case, causal, D, dtype):
    """Run fa_bwd (caller workspace) and fa_bwd_noalloc on one problem."""
    q, k, v, do = (case[n].cuda() for n in ("q", "k", "v", "do"))
    B, Sq, H, _ = q.shape
    Sk = k.shape[1]
    scale = D ** -0.5
    dt = fa.FA_BF16 if dtype == torch.bfloat16 else fa.FA_FP16
    o, lse = fa.forward(q, k, v, causal=causal, scale=scale)
    ref = [torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)]
    ws = fa.workspace_for(B, H, Sq, D, q.device)
    stream = torch.cuda.current_stream().cuda_stream
    st = fa.fa_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(do), *(_ptr(t) for t in ref),
                   B, H, Sq, Sk, D, scale, int(causal), dt, _ptr(ws), ws.numel(), stream)
    assert st == 0, fa.fa_strerror(st)
    new = [torch.full_like(q, float("nan")), torch.full_like(k, float("nan")), torch.full_like(v, float("nan"))]
    st = fa.fa_bwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(do), *(_ptr(t) for t in new),
                           B, H, Sq, Sk, D, scale, int(causal), dt, stream)
    assert st == 0, fa.fa_strerror(st)
    torch.cuda.synchronize()
    status, detail = fa.fa_last_device_status()
    assert status == 0, (status, detail)
    return ref, new


@pytest.mark.gpu
def test_noalloc_matches_fa_bwd_on_two_calls_in_a_row(fa_lib):
    # First call: a larger problem; second call: a smaller one with another
    # head_dim and dtype, which reads scratch the first call wrote. Both entry
    # points run the same kernels: dK and dV come out bit-identical, and dQ,
    # summed with fp32 atomics in whatever order the blocks finish, agrees to
    # well within 1e-3. The first call is also checked against the oracle.
    calls = [
        (random_case(2, 4, 1000, 1000, 128, torch.bfloat16, 101), True, 128, torch.bfloat16),
        (random_case(1, 3, 333, 517, 64, torch.float16, 102), False, 64, torch.float16),
    ]
    for n_call, (case, causal, D, dtype) in enumerate(calls):
        ref, new = _bwd_both(case, causal, D, dtype)
        for name, r, x in zip(("dq", "dk", "dv"), ref, new):
            assert torch.isfinite(x).all(), name
            if name == "dq":
                err = rel_l2(np64(x), np64(r))
                assert err <= 1e-3, f"call {n_call} dq: relative L2 {err:.3e} vs fa_bwd"
            else:
                assert torch.equal(x, r), f"call {n_call} {name}: differs from fa_bwd"
        if n_call == 0:
            qn, kn, vn, don = (np64(case[n]) for n in ("q", "k", "v", "do"))
            dq_r, dk_r, dv_r, _ = oracle.attention_backward(qn, kn, vn, don, D ** -0.5, causal)
            for name, g, r in (("dq", new[0], dq_r), ("dk", new[1], dk_r), ("dv", new[2], dv_r)):
                check_grad(np64(g), r, f"noalloc {name}", row_axis=1, head_axes=(0, 2))


@pytest.mark.gpu
def test_noalloc_torch_helper(fa_lib):
    """backward_noalloc (the torch helper) on the device of q, against fa_bwd."""
    case = random_case(1, 2, 300, 300, 64, torch.bfloat16, 103)
    q, k, v, do = (case[n].cuda() for n in ("q", "k", "v", "do"))
    o, lse = fa.forward(q, k, v, causal=True)
    dq, dk, dv = fa.backward_noalloc(q, k, v, o, lse, do, causal=True)
    rq, rk, rv = fa.backward(q, k, v, o, lse, do, causal=True)
    torch.cuda.synchronize()
    assert fa.fa_last_device_status()[0] == 0
    assert torch.equal(dk, rk) and torch.equal(dv, rv)
    assert rel_l2(np64(dq), np64(rq)) <= 1e-3


def test_noalloc_rejects_problems_beyond_its_scratch(fa_lib):
    # B*H*Sq_pad*(D+2)*4 bytes = 16*16384*130*4 = 136 MB > 64 MiB
    st = fa.fa_bwd_noalloc(A, A, A, A, A, A, A, A, A, 1, 16, 16384, 16384, 128, 0.088, 1, fa.FA_BF16, 0)
    assert st == -8
    assert "64 MiB" in fa.fa_strerror(st)
    # the ordinary argument checks still come first
    assert fa.fa_bwd_noalloc(None, A, A, A, A, A, A, A, A, 1, 1, 8, 8, 64, 0.1, 0, fa.FA_FP16, 0) == -1
    assert fa.fa_bwd_noalloc(A, A, A, A, A, A, A, A, A, 1, 1, 8, 8, 100, 0.1, 0, fa.FA_FP16, 0) == -2
