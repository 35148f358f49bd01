"""The check build (libfa_check.so: the same kernels compiled with FA_CHECK=1,
device-side index and bounds checks that record FA_ERR_BOUNDS and skip the
access) on ragged, rectangular, narrow-head, deterministic and e4m3 cases.
Every call must match the oracle as the normal build does, and leave the
device status word clear: no check failed."""
import os

import numpy as np
import pytest
import torch

import oracle
import oracle.fp8
from exact_io_aware_96_b200 import build, fa
from exact_io_aware_96_b200.inputs import quantize_e4m3, random_case
from tests.parity import check_fp8_o_lse, check_o_lse, full_check, np64, rel_l2

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def check_lib():
    if not os.path.exists(fa.LIB_CHECK_PATH):
        build.build(check=True)
    normal = fa.LIB_PATH
    fa.use_library(fa.LIB_CHECK_PATH)
    try:
        yield fa.lib()
    finally:
        fa.use_library(normal)


def _status_clear(what):
    st, detail = fa.fa_last_device_status()
    assert st == 0, f"{what}: device status {fa.STATUS.get(st, st)} {detail} (check site = detail[3])"


CASES = [  # B, H, Sq, Sk, D, dtype, causal
    (1, 2, 1, 1, 64, torch.float16, False),
    (2, 3, 129, 700, 128, torch.bfloat16, True),
    (2, 3, 700, 129, 64, torch.float16, True),
    (1, 2, 300, 257, 40, torch.bfloat16, True),
    (1, 2, 257, 300, 96, torch.float16, False),
    (2, 2, 640, 640, 128, torch.bfloat16, True),
    (1, 1, 2000, 2000, 64, torch.float16, True),
    (1, 2, 513, 255, 128, torch.bfloat16, False),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"B{c[0]}H{c[1]}Sq{c[2]}Sk{c[3]}D{c[4]}c{int(c[6])}")
def test_check_build_forward_backward(check_lib, case):
    B, H, Sq, Sk, D, dtype, causal = case
    c = random_case(B, H, Sq, Sk, D, dtype, 700 + Sq + D)
    full_check(c, causal, what=f"check build {case}")
    _status_clear(str(case))


@pytest.mark.parametrize("D,causal", [(64, True), (128, False)])
def test_check_build_deterministic(check_lib, D, causal):
    c = random_case(1, 2, 300, 257, D, torch.bfloat16, 800 + D)
    q, k, v, do = (c[n].cuda() for n in ("q", "k", "v", "do"))
    o, lse = fa.forward(q, k, v, causal=causal)
    det = fa.backward(q, k, v, o, lse, do, causal=causal, deterministic=True)
    ato = fa.backward(q, k, v, o, lse, do, causal=causal)
    torch.cuda.synchronize()
    _status_clear(f"deterministic D{D}")
    assert torch.equal(det[1], ato[1]) and torch.equal(det[2], ato[2])
    assert rel_l2(np64(det[0]), np64(ato[0])) < 2e-3


@pytest.mark.parametrize("Sq,Sk,causal", [(300, 257, True), (129, 700, False)])
def test_check_build_e4m3(check_lib, Sq, Sk, causal):
    c = random_case(1, 2, Sq, Sk, 128, torch.bfloat16, 900 + Sq)
    z = {n: quantize_e4m3(c[n].float()) for n in ("q", "k", "v")}
    o, lse = fa.forward_fp8(*(z[n][0].cuda() for n in ("q", "k", "v")), *(z[n][1] for n in ("q", "k", "v")),
                            causal=causal)
    torch.cuda.synchronize()
    _status_clear("e4m3")
    dq8 = {n: oracle.fp8.dequantize(z[n][0].numpy(), z[n][1]) for n in ("q", "k", "v")}
    for h in range(2):
        rows = np.arange(Sq)
        check_fp8_o_lse(np64(o)[0, :, h], np64(lse)[0, h], dq8["q"], dq8["k"], dq8["v"], 128 ** -0.5, causal,
                        torch.bfloat16, 0, h, rows, f"check build e4m3 h{h}")


@pytest.mark.parametrize("Sq,Sk,D,causal", [(1000, 1000, 128, True), (700, 129, 64, True), (513, 300, 96, False),
                                            (300, 1, 64, False)])
def test_check_build_split_forward(check_lib, Sq, Sk, D, causal):
    """The forward with every query-block rank split by key range (the
    workspace slots, the tickets and the unit order are all checked sites)."""
    c = random_case(2, 3, Sq, Sk, D, torch.bfloat16, 950 + Sq + D)
    q, k, v = (c[n].cuda() for n in ("q", "k", "v"))
    n, ns = fa.fwd_workspace_size(2, 3, Sq, Sk, D, causal, 64)
    assert ns == (Sq + 255) // 256
    ws = torch.full((n,), 255, dtype=torch.uint8, device="cuda")
    o, lse = fa.forward(q, k, v, causal=causal, split_ranks=64, workspace=ws)
    torch.cuda.synchronize()
    _status_clear(f"split forward Sq{Sq} Sk{Sk} D{D}")
    o_ref, lse_ref = oracle.attention_forward(np64(c["q"]), np64(c["k"]), np64(c["v"]), D ** -0.5, causal)
    check_o_lse(np64(o), np64(lse), o_ref, lse_ref, torch.bfloat16, f"check build split Sq{Sq} Sk{Sk} D{D}")
