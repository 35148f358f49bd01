"""HostAttentionPipeline: pinned host buffers in, pinned host buffers out,
copies overlapped with the neighbouring steps' kernels. Every step's results
must equal those of the plain device calls on the same inputs."""
import pytest
import torch

from exact_io_aware_96_b200 import fa
from exact_io_aware_96_b200.host_pipeline import HostAttentionPipeline
from exact_io_aware_96_b200.inputs import random_case
from tests.parity import np64, rel_l2

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("depth", [1, 2, 3])
def test_pipeline_matches_device_calls(depth):
    B, H, S, D = 1, 4, 1000, 128
    steps = 5
    cases = [random_case(B, H, S, S, D, torch.bfloat16, 700 + i) for i in range(steps)]
    pin = lambda t: t.contiguous().pin_memory()  # noqa: E731
    ins = [{n: pin(c[n]) for n in ("q", "k", "v", "do")} for c in cases]
    outs = [{"o": torch.empty(B, S, H, D, dtype=torch.bfloat16).pin_memory(),
             "lse": torch.empty(B, H, S, dtype=torch.float32).pin_memory(),
             **{n: torch.empty(B, S, H, D, dtype=torch.bfloat16).pin_memory() for n in ("dq", "dk", "dv")}}
            for _ in range(steps)]
    pipe = HostAttentionPipeline(B, S, H, D, dtype=torch.bfloat16, causal=True, depth=depth)
    for i in range(steps):
        x, y = ins[i], outs[i]
        pipe.step(x["q"], x["k"], x["v"], x["do"], y["o"], y["lse"], y["dq"], y["dk"], y["dv"])
    pipe.synchronize()
    assert fa.fa_last_device_status()[0] == 0
    for i in range(steps):
        q, k, v, do = (cases[i][n].cuda() for n in ("q", "k", "v", "do"))
        o, lse = fa.forward(q, k, v, causal=True)
        dq, dk, dv = fa.backward(q, k, v, o, lse, do, causal=True)
        torch.cuda.synchronize()
        assert torch.equal(outs[i]["o"], o.cpu()) and torch.equal(outs[i]["lse"], lse.cpu())
        assert torch.equal(outs[i]["dk"], dk.cpu()) and torch.equal(outs[i]["dv"], dv.cpu())
        assert rel_l2(np64(outs[i]["dq"]), np64(dq)) < 1e-3   # dq: atomic summation order


def test_pipeline_rejects_pageable_and_misshaped_buffers():
    B, H, S, D = 1, 2, 256, 64
    pipe = HostAttentionPipeline(B, S, H, D, dtype=torch.float16)
    good = lambda: torch.zeros(B, S, H, D, dtype=torch.float16).pin_memory()  # noqa: E731
    lse = torch.zeros(B, H, S, dtype=torch.float32).pin_memory()
    with pytest.raises(ValueError):
        pipe.step(torch.zeros(B, S, H, D, dtype=torch.float16), good(), good(), good(), good(), lse,
                  good(), good(), good())
    with pytest.raises(ValueError):
        pipe.step(good(), good(), good(), good(), good(), torch.zeros(B, S, H, dtype=torch.float32).pin_memory(),
                  good(), good(), good())
