"""Out-of-bounds writes, caught without a sanitizer: every output the kernels
write (O, LSE, dQ, dK, dV, the e4m3 forward's O and LSE) lives inside one
larger device buffer whose margins before and after hold a canary byte
pattern; after the calls the margins must be unchanged, and the outputs must
still match the oracle. Ragged lengths, head dims below the kernel width and
strided views are where a stray store would land."""
import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_96_b200 import fa
from exact_io_aware_96_b200.inputs import quantize_e4m3, random_case
from tests.parity import check_grad, check_o_lse, np64

pytestmark = pytest.mark.gpu

CANARY = 0xA5
MARGIN = 1 << 16  # bytes on each side


class Guarded:
    """A device tensor of `shape`/`dtype` placed MARGIN bytes into a canary-filled buffer."""

    def __init__(self, shape, dtype, fill=float("nan")):
        n = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
        self.raw = torch.full((MARGIN + n + MARGIN,), CANARY, dtype=torch.uint8, device="cuda")
        self.t = self.raw[MARGIN:MARGIN + n].view(dtype).view(shape)
        if dtype.is_floating_point:
            self.t.fill_(fill)

    def margins_intact(self):
        return bool((self.raw[:MARGIN] == CANARY).all()) and bool((self.raw[-MARGIN:] == CANARY).all())


def _run(B, H, Sq, Sk, D, dtype, causal, seed, deterministic=False):
    c = random_case(B, H, Sq, Sk, D, dtype, seed)
    q, k, v, do = (c[n].cuda() for n in ("q", "k", "v", "do"))
    o = Guarded((B, Sq, H, D), dtype)
    lse = Guarded((B, H, Sq), torch.float32)
    dq, dk, dv = Guarded((B, Sq, H, D), dtype), Guarded((B, Sk, H, D), dtype), Guarded((B, Sk, H, D), dtype)
    ws = fa.workspace_for(B, H, Sq, D, q.device, Sk=Sk, deterministic=deterministic)
    ws_g = torch.full((MARGIN + ws.numel() + MARGIN,), CANARY, dtype=torch.uint8, device="cuda")
    ws_view = ws_g[MARGIN:MARGIN + ws.numel()]
    fa.forward(q, k, v, causal=causal, out=o.t, lse=lse.t)
    fa.backward(q, k, v, o.t, lse.t, do, causal=causal, dq=dq.t, dk=dk.t, dv=dv.t, workspace=ws_view,
                deterministic=deterministic)
    torch.cuda.synchronize()
    assert fa.fa_last_device_status()[0] == 0
    what = f"B{B} H{H} Sq{Sq} Sk{Sk} D{D} c{causal} det{deterministic}"
    for name, g in (("o", o), ("lse", lse), ("dq", dq), ("dk", dk), ("dv", dv)):
        assert g.margins_intact(), f"{what}: write outside {name}"
    assert bool((ws_g[:MARGIN] == CANARY).all()) and bool((ws_g[-MARGIN:] == CANARY).all()), \
        f"{what}: write outside the workspace"
    sc = D ** -0.5
    qn, kn, vn, don = (np64(c[n]) for n in ("q", "k", "v", "do"))
    o_ref, lse_ref = oracle.attention_forward(qn, kn, vn, sc, causal)
    check_o_lse(np64(o.t), np64(lse.t), o_ref, lse_ref, dtype, what)
    dq_r, dk_r, dv_r, _ = oracle.attention_backward(qn, kn, vn, don, sc, causal)
    for name, g, r in (("dq", dq, dq_r), ("dk", dk, dk_r), ("dv", dv, dv_r)):
        check_grad(np64(g.t), r, f"{what} {name}", row_axis=1, head_axes=(0, 2))


@pytest.mark.parametrize("Sq,Sk", [(1, 1), (129, 129), (300, 257), (257, 300), (700, 129)])
@pytest.mark.parametrize("D", [40, 64, 96, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_no_write_outside_outputs(Sq, Sk, D, causal):
    _run(1, 3, Sq, Sk, D, torch.bfloat16, causal, seed=Sq * 7 + Sk + D)


@pytest.mark.parametrize("D", [64, 128])
def test_no_write_outside_outputs_deterministic(D):
    _run(2, 2, 333, 300, D, torch.float16, True, seed=99 + D, deterministic=True)


@pytest.mark.parametrize("Sq,Sk,D", [(1, 1, 16), (129, 200, 48), (300, 257, 128)])
def test_no_write_outside_outputs_e4m3(Sq, Sk, D):
    B, H = 1, 2
    c = random_case(B, H, Sq, Sk, D, torch.float32, 5 + Sq)
    z = {n: quantize_e4m3(c[n]) for n in ("q", "k", "v")}
    o = Guarded((B, Sq, H, D), torch.bfloat16)
    lse = Guarded((B, H, Sq), torch.float32)
    fa.forward_fp8(*(z[n][0].cuda() for n in ("q", "k", "v")), *(z[n][1] for n in ("q", "k", "v")),
                   causal=True, out=o.t, lse=lse.t)
    torch.cuda.synchronize()
    assert fa.fa_last_device_status()[0] == 0
    assert o.margins_intact() and lse.margins_intact()
    assert bool(torch.isfinite(o.t).all())
