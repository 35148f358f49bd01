"""Forward parity on the GPU: libfa.so (through the C ABI) vs the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_96_b200 import fa
from exact_io_aware_96_b200.inputs import WORKLOADS, make_inputs, random_case, sample_rows
from tests.parity import check_o_lse, np64, run_fwd

pytestmark = pytest.mark.gpu


def _fwd_case(B, H, Sq, Sk, D, dtype, causal, seed, scale=None, qk_std=1.0):
    c = random_case(B, H, Sq, Sk, D, dtype, seed, qk_std)
    sc = D ** -0.5 if scale is None else scale
    o, lse = run_fwd(c["q"].cuda(), c["k"].cuda(), c["v"].cuda(), causal, sc)
    o_ref, lse_ref = oracle.attention_forward(np64(c["q"]), np64(c["k"]), np64(c["v"]), sc, causal)
    check_o_lse(np64(o), np64(lse), o_ref, lse_ref, dtype, f"B{B} H{H} Sq{Sq} Sk{Sk} D{D} {dtype} c{causal}")


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("S", [1, 7, 63, 65, 127, 128, 129, 255, 256, 257, 640])
def test_fwd_square(D, dtype, causal, S):
    _fwd_case(1, 2, S, S, D, dtype, causal, seed=1000 + S)


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("Sq,Sk", [(1, 300), (100, 37), (129, 700), (700, 129), (300, 1), (256, 512), (513, 255)])
def test_fwd_rectangular(D, causal, Sq, Sk):
    # causal with Sq > Sk leaves the first Sq - Sk rows with no key: O = 0, LSE = -inf
    _fwd_case(2, 3, Sq, Sk, D, torch.bfloat16, causal, seed=7 + Sq + Sk)


@pytest.mark.parametrize("D", [8, 32, 40, 72, 96, 120])
@pytest.mark.parametrize("causal", [False, True])
def test_fwd_other_head_dims(D, causal):
    # head_dim below the kernel width: the extra columns are read as zeros
    _fwd_case(2, 2, 300, 257, D, torch.bfloat16, causal, seed=90 + D, scale=D ** -0.5)


@pytest.mark.parametrize("scale", [0.01, 0.5, 1.0])
def test_fwd_scale(scale):
    _fwd_case(1, 2, 300, 300, 64, torch.float16, True, seed=5, scale=scale)


def test_fwd_wide_scores():
    # Q, K ~ N(0, 2^2): scores spread wide, the running max is raised often
    _fwd_case(1, 2, 1000, 1000, 128, torch.bfloat16, False, seed=11, qk_std=2.0)
    _fwd_case(1, 2, 1000, 1000, 128, torch.bfloat16, True, seed=12, qk_std=4.0)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("qk_std", [3.0, 6.0])
@pytest.mark.parametrize("S", [300, 1000, 1500])
def test_fwd_wide_scores_d64(causal, qk_std, S):
    """D = 64 rescales O_t while later S products are already in flight (three
    rotating S buffers): the running max must be raised on the last and the
    middle blocks of a tile alike."""
    _fwd_case(2, 2, S, S, 64, torch.float16, causal, seed=int(13 * qk_std) + S, qk_std=qk_std)


def test_fwd_repeatable():
    c = random_case(1, 4, 777, 777, 128, torch.bfloat16, 3)
    q, k, v = c["q"].cuda(), c["k"].cuda(), c["v"].cuda()
    o1, l1 = run_fwd(q, k, v, True)
    o2, l2 = run_fwd(q, k, v, True)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


@pytest.mark.parametrize("name", ["c1", "c2", "c3", "c3r"])
def test_fwd_workloads_full(name):
    w = WORKLOADS[name]
    inp = make_inputs(w)
    for causal in w.causal:
        q, k, v = inp["q"].cuda(), inp["k"].cuda(), inp["v"].cuda()
        if w.packed:
            qkv = inp["qkv"].cuda()
            q, k, v = qkv[:, :, 0], qkv[:, :, 1], qkv[:, :, 2]   # strided views into [B,S,3,H,D]
        o, lse = run_fwd(q, k, v, causal, w.scale)
        o_ref, lse_ref = oracle.attention_forward(np64(inp["q"]), np64(inp["k"]), np64(inp["v"]), w.scale, causal)
        check_o_lse(np64(o), np64(lse), o_ref, lse_ref, w.dtype, f"{name} causal={causal}")


@pytest.mark.parametrize("name", ["c4", "c5"])
def test_fwd_workloads_sampled(name):
    """Full-size launch; O and LSE checked on sampled rows of every head."""
    w = WORKLOADS[name]
    inp = make_inputs(w)
    q, k, v = inp["q"].cuda(), inp["k"].cuda(), inp["v"].cuda()
    rows = sample_rows(w.S, 128, 246 if name == "c5" else 118, w.seed)
    qn, kn, vn = np64(inp["q"]), np64(inp["k"]), np64(inp["v"])
    for causal in w.causal:
        o, lse = run_fwd(q, k, v, causal, w.scale)
        o, lse = np64(o), np64(lse)
        for h in range(w.H):
            o_ref, lse_ref = oracle.attention_forward_rows(qn, kn, vn, w.scale, causal, 0, h, rows)
            check_o_lse(o[0, rows, h], lse[0, h, rows], o_ref, lse_ref, w.dtype, f"{name} h{h} causal={causal}")


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
def test_fwd_masked_keys_weigh_zero(D, dtype):
    """Causal: keys past a row's diagonal must get P exactly 0, not a tiny
    weight. V on keys >= T is set to the largest power of two of the format
    (2^127 in bf16, 2^15 in fp16): rows below T, which never see those keys,
    must match the oracle and be bit-identical to a run with those V rows 0.
    T = 448 cuts through the diagonal block of the second 256-row query
    block, so element-wise masking is exercised."""
    S, T = 512, 448
    c = random_case(1, 2, S, S, D, dtype, 31 + D)
    big = 2.0 ** 127 if dtype == torch.bfloat16 else 2.0 ** 15
    v_big, v_zero = c["v"].clone(), c["v"].clone()
    v_big[:, T:] = big
    v_zero[:, T:] = 0
    q, k = c["q"].cuda(), c["k"].cuda()
    o_big, lse_big = run_fwd(q, k, v_big.cuda(), True)
    o_zero, lse_zero = run_fwd(q, k, v_zero.cuda(), True)
    assert torch.equal(o_big[:, :T], o_zero[:, :T]), "masked keys leaked into O"
    assert torch.equal(lse_big, lse_zero)
    o_ref, lse_ref = oracle.attention_forward(np64(c["q"]), np64(c["k"]), np64(v_big), D ** -0.5, True)
    check_o_lse(np64(o_big[:, :T]), np64(lse_big), o_ref[:, :T], lse_ref, dtype, f"D{D} {dtype} huge masked V")
