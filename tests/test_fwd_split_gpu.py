"""Forward with the key-range split (fa_fwd_params.workspace / split_ranks):
the heaviest query blocks run as two CTAs, one per half of the key blocks,
whose partial (m, l, unnormalised O) merge exactly in the CTA that finishes
second. Checked against the fp64 oracle on forced and automatic splits, for
repeatability (the merge is symmetric in its two halves, so the result does
not depend on which CTA finishes first), for agreement with the unsplit
kernel, and for workspace reuse and garbage-filled workspaces."""
import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_96_b200 import fa
from exact_io_aware_96_b200.inputs import WORKLOADS, make_inputs, random_case, sample_rows
from tests.parity import check_o_lse, np64

pytestmark = pytest.mark.gpu


def _run(q, k, v, causal, split_ranks, workspace=None, scale=None):
    o, lse = fa.forward(q, k, v, causal=causal, scale=scale, split_ranks=split_ranks, workspace=workspace)
    torch.cuda.synchronize()
    st, detail = fa.fa_last_device_status()
    assert st == 0, f"device status {st} {detail}"
    return o, lse


def _case(B, H, Sq, Sk, D, dtype, causal, split_ranks, seed):
    c = random_case(B, H, Sq, Sk, D, dtype, seed)
    q, k, v = c["q"].cuda(), c["k"].cuda(), c["v"].cuda()
    n, ns = fa.fwd_workspace_size(B, H, Sq, Sk, D, causal, split_ranks)
    assert ns == min(split_ranks, (Sq + 255) // 256) and n > 0
    o, lse = _run(q, k, v, causal, split_ranks)
    o_ref, lse_ref = oracle.attention_forward(np64(c["q"]), np64(c["k"]), np64(c["v"]), D ** -0.5, causal)
    check_o_lse(np64(o), np64(lse), o_ref, lse_ref, dtype, f"split {split_ranks} B{B} H{H} Sq{Sq} Sk{Sk} D{D} c{causal}")
    return q, k, v, o, lse


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("S", [1, 129, 257, 300, 640, 1000])
@pytest.mark.parametrize("split_ranks", [1, 64])
def test_split_square(D, dtype, causal, S, split_ranks):
    _case(2, 2, S, S, D, dtype, causal, split_ranks, seed=3000 + S + D)


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("Sq,Sk", [(129, 700), (700, 129), (513, 255), (300, 1), (1, 300), (256, 1024)])
def test_split_rectangular(D, causal, Sq, Sk):
    # causal with Sq > Sk: rows with no key in either half (O = 0, LSE = -inf)
    _case(1, 3, Sq, Sk, D, torch.bfloat16, causal, 64, seed=41 + Sq + Sk)


@pytest.mark.parametrize("D", [40, 96])
def test_split_narrow_head(D):
    _case(1, 2, 600, 600, D, torch.float16, True, 64, seed=77 + D)


def test_split_wide_scores():
    # Q, K ~ N(0, 4^2): the two halves' row maxima differ widely
    c = random_case(1, 2, 1000, 1000, 128, torch.bfloat16, 13, qk_std=4.0)
    q, k, v = c["q"].cuda(), c["k"].cuda(), c["v"].cuda()
    for causal in (False, True):
        o, lse = _run(q, k, v, causal, 64)
        o_ref, lse_ref = oracle.attention_forward(np64(c["q"]), np64(c["k"]), np64(c["v"]), 128 ** -0.5, causal)
        check_o_lse(np64(o), np64(lse), o_ref, lse_ref, torch.bfloat16, f"wide scores causal={causal}")


@pytest.mark.parametrize("D,causal", [(64, False), (128, True)])
def test_split_repeatable_and_close_to_unsplit(D, causal):
    c = random_case(2, 3, 1000, 1000, D, torch.bfloat16, 5 + D)
    q, k, v = c["q"].cuda(), c["k"].cuda(), c["v"].cuda()
    o1, l1 = _run(q, k, v, causal, 64)
    for _ in range(3):
        o2, l2 = _run(q, k, v, causal, 64)
        assert torch.equal(o1, o2) and torch.equal(l1, l2), "split result depends on which CTA merges"
    o0, l0 = _run(q, k, v, causal, -1)
    # Same exact attention, different rounding order: O within a few bf16
    # ulps; LSE within 1e-4, the worst-case relative error of an fp32 row sum
    # over 1000 terms (1000 x 2^-24 = 6e-5) plus the merge factors' ex2
    # approximation, and ten times below the oracle tolerance.
    assert (o1.float() - o0.float()).abs().max().item() <= 2 ** -6
    assert (l1 - l0).abs().max().item() <= 1e-4


def test_split_workspace_reuse_and_garbage():
    """One workspace for consecutive calls of different shapes (each launch
    has its own epoch, so tickets left by the previous call do not pair with
    this one), and a workspace filled with 0xff bytes before first use."""
    n = max(fa.fwd_workspace_size(2, 4, S, S, 128, True, 64)[0] for S in (640, 1000))
    ws = torch.full((n,), 255, dtype=torch.uint8, device="cuda")
    for S, causal, seed in ((1000, True, 1), (640, False, 2), (1000, True, 3), (640, True, 4)):
        c = random_case(2, 4, S, S, 128, torch.bfloat16, seed)
        o, lse = _run(c["q"].cuda(), c["k"].cuda(), c["v"].cuda(), causal, 64, workspace=ws)
        o_ref, lse_ref = oracle.attention_forward(np64(c["q"]), np64(c["k"]), np64(c["v"]), 128 ** -0.5, causal)
        check_o_lse(np64(o), np64(lse), o_ref, lse_ref, torch.bfloat16, f"reuse S{S} causal={causal}")


def test_split_workspace_errors():
    c = random_case(1, 2, 640, 640, 128, torch.bfloat16, 9)
    q, k, v = c["q"].cuda(), c["k"].cuda(), c["v"].cuda()
    n, ns = fa.fwd_workspace_size(1, 2, 640, 640, 128, True, 64)
    assert ns == 3
    small = torch.empty(n - 256, dtype=torch.uint8, device="cuda")
    with pytest.raises(fa.FaError) as e:
        fa.forward(q, k, v, causal=True, split_ranks=64, workspace=small)
    assert e.value.status == fa.FA_ERR_WORKSPACE
    big = torch.empty(n + 512, dtype=torch.uint8, device="cuda")
    with pytest.raises(fa.FaError) as e:
        fa.forward(q, k, v, causal=True, split_ranks=64, workspace=big[16:])
    assert e.value.status == fa.FA_ERR_MISALIGNED


@pytest.mark.parametrize("name", ["c2", "c3", "c3r", "c4"])
def test_split_automatic_workloads(name):
    """The library's own choice on the small-grid workloads: these are the
    shapes where B * H * ceil(S / 256) leaves SMs idle."""
    w = WORKLOADS[name]
    inp = make_inputs(w)
    q, k, v = inp["q"].cuda(), inp["k"].cuda(), inp["v"].cuda()
    if w.packed:
        qkv = inp["qkv"].cuda()
        q, k, v = qkv[:, :, 0], qkv[:, :, 1], qkv[:, :, 2]
    qn, kn, vn = np64(inp["q"]), np64(inp["k"]), np64(inp["v"])
    for causal in w.causal:
        n, ns = fa.fwd_workspace_size(w.B, w.H, w.S, w.S, w.D, causal, 0)
        assert (n > 0) == (ns > 0)
        o, lse = _run(q, k, v, causal, 0)
        if name == "c4":
            rows = sample_rows(w.S, 128, 118, w.seed)
            o, lse = np64(o), np64(lse)
            for h in range(w.H):
                o_ref, lse_ref = oracle.attention_forward_rows(qn, kn, vn, w.scale, causal, 0, h, rows)
                check_o_lse(o[0, rows, h], lse[0, h, rows], o_ref, lse_ref, w.dtype, f"{name} h{h} n_split={ns}")
        else:
            o_ref, lse_ref = oracle.attention_forward(qn, kn, vn, w.scale, causal)
            check_o_lse(np64(o), np64(lse), o_ref, lse_ref, w.dtype, f"{name} causal={causal} n_split={ns}")


def test_split_not_chosen_for_many_waves():
    # c5: 1024 CTAs on 148 SMs, the tail is already short
    w = WORKLOADS["c5"]
    for causal in w.causal:
        assert fa.fwd_workspace_size(w.B, w.H, w.S, w.S, w.D, causal, 0) == (0, 0)
