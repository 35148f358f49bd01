"""Failure detection on the GPU without a fault: a pipeline wait that nothing
completes runs out after its limit, the status word records it, and the
context stays usable for ordinary calls."""
import time

import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_96_b200 import fa
from exact_io_aware_96_b200.inputs import random_case
from tests.parity import check_o_lse, np64, run_fwd

pytestmark = pytest.mark.gpu


def test_wait_timeout_is_recorded_and_context_survives():
    torch.cuda.synchronize()
    assert fa.fa_last_device_status()[0] == 0            # clean start (and cleared)
    t0 = time.perf_counter()
    assert fa.fa_selftest_wait_timeout(20000) == 0      # 20 ms limit
    st, detail = fa.fa_last_device_status()             # synchronises
    dt = time.perf_counter() - t0
    assert st == -5 and fa.STATUS[st] == "FA_ERR_TIMEOUT"
    assert detail == [-5, 0, 4, 0]                      # code, block 0, role self-test, iteration 0
    assert dt >= 0.02
    assert fa.fa_last_device_status()[0] == 0            # reading cleared it
    # the context still runs the attention kernels correctly
    c = random_case(1, 2, 257, 257, 64, torch.float16, 5)
    o, lse = run_fwd(c["q"].cuda(), c["k"].cuda(), c["v"].cuda(), True)
    o_ref, lse_ref = oracle.attention_forward(np64(c["q"]), np64(c["k"]), np64(c["v"]), 64 ** -0.5, True)
    check_o_lse(np64(o), np64(lse), o_ref, lse_ref, torch.float16, "after self-test")


def test_wait_timeout_on_a_side_stream():
    s = torch.cuda.Stream()
    assert fa.fa_selftest_wait_timeout(1000, s.cuda_stream) == 0
    s.synchronize()
    st, detail = fa.fa_last_device_status()
    assert st == -5 and detail[2] == 4
