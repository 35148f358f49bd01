"""Backward parity on the GPU: libfa.so (through the C ABI) vs the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_96_b200 import fa
from exact_io_aware_96_b200.inputs import WORKLOADS, make_inputs, random_case, sample_rows
from tests.parity import check_grad, check_o_lse, full_check, np64, rel_l2, run_bwd, run_fwd

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("S", [1, 7, 63, 64, 65, 127, 128, 129, 200, 256, 257, 640])
def test_bwd_square(D, dtype, causal, S):
    full_check(random_case(1, 2, S, S, D, dtype, 2000 + S), causal, what=f"S{S} D{D} {dtype} c{causal}")


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("Sq,Sk", [(1, 300), (100, 37), (129, 700), (700, 129), (300, 1), (256, 512), (513, 255)])
def test_bwd_rectangular(D, causal, Sq, Sk):
    full_check(random_case(2, 3, Sq, Sk, D, torch.bfloat16, 31 + Sq + Sk), causal,
               what=f"Sq{Sq} Sk{Sk} D{D} c{causal}")


@pytest.mark.parametrize("D", [8, 32, 40, 72, 96, 120])
@pytest.mark.parametrize("causal", [False, True])
def test_bwd_other_head_dims(D, causal):
    full_check(random_case(2, 2, 300, 257, D, torch.float16, 190 + D), causal, what=f"D{D} c{causal}")


@pytest.mark.parametrize("scale", [0.02, 0.5])
def test_bwd_scale(scale):
    full_check(random_case(1, 2, 300, 300, 128, torch.float16, 9), True, scale=scale, what=f"scale {scale}")


def test_bwd_wide_scores():
    full_check(random_case(1, 2, 700, 700, 128, torch.bfloat16, 13, qk_std=2.0), True, what="wide")


@pytest.mark.parametrize("name", ["c1", "c3", "c3r"])
def test_bwd_workloads_full(name):
    w = WORKLOADS[name]
    inp = make_inputs(w)
    for causal in w.causal:
        full_check(inp, causal, scale=w.scale, what=f"{name} causal={causal}")


def test_bwd_packed_qkv():
    """c2: q, k, v are strided views into one [B, S, 3, H, D] tensor; the
    gradients are written into the matching views of one dqkv tensor."""
    w = WORKLOADS["c2"]
    inp = make_inputs(w)
    qkv = inp["qkv"].cuda()
    do = inp["do"].cuda()
    q, k, v = qkv[:, :, 0], qkv[:, :, 1], qkv[:, :, 2]
    o, lse = run_fwd(q, k, v, False, w.scale)
    dqkv = torch.full_like(qkv, float("nan"))
    fa.backward(q, k, v, o, lse, do, causal=False, scale=w.scale,
                dq=dqkv[:, :, 0], dk=dqkv[:, :, 1], dv=dqkv[:, :, 2])
    torch.cuda.synchronize()
    qn, kn, vn, don = np64(inp["q"]), np64(inp["k"]), np64(inp["v"]), np64(inp["do"])
    o_ref, lse_ref = oracle.attention_forward(qn, kn, vn, w.scale, False)
    check_o_lse(np64(o), np64(lse), o_ref, lse_ref, w.dtype, "c2 fwd")
    dq_r, dk_r, dv_r, _ = oracle.attention_backward(qn, kn, vn, don, w.scale, False)
    g = np64(dqkv)
    for j, (name, ref) in enumerate((("dq", dq_r), ("dk", dk_r), ("dv", dv_r))):
        check_grad(g[:, :, j], ref, f"c2 {name}", row_axis=1, head_axes=(0, 2))


def test_bwd_repeatable_dk_dv():
    """dK and dV have a fixed summation order; dQ is accumulated with atomics."""
    c = random_case(1, 2, 900, 900, 128, torch.bfloat16, 17)
    q, k, v, do = (c[n].cuda() for n in ("q", "k", "v", "do"))
    o, lse = run_fwd(q, k, v, True)
    a = run_bwd(q, k, v, o, lse, do, True)
    b = run_bwd(q, k, v, o, lse, do, True)
    assert torch.equal(a[1], b[1]) and torch.equal(a[2], b[2])
    assert rel_l2(np64(a[0]), np64(b[0])) < 1e-3


@pytest.mark.parametrize("name", ["c4", "c5"])
def test_bwd_workloads_sampled(name):
    """Full-size launch. dQ checked on sampled rows of every head; dK and dV
    need every query row, so they are checked in full on the first and last head."""
    w = WORKLOADS[name]
    inp = make_inputs(w)
    dev = {n: inp[n].cuda() for n in ("q", "k", "v", "do")}
    rows = sample_rows(w.S, 128, 246 if name == "c5" else 118, w.seed)
    qn, kn, vn, don = (np64(inp[n]) for n in ("q", "k", "v", "do"))
    for causal in w.causal:
        o, lse = run_fwd(dev["q"], dev["k"], dev["v"], causal, w.scale)
        dq, dk, dv = run_bwd(dev["q"], dev["k"], dev["v"], o, lse, dev["do"], causal, w.scale)
        dq, dk, dv = np64(dq), np64(dk), np64(dv)
        got, ref = [], []
        for h in range(w.H):
            got.append(dq[0, rows, h])
            ref.append(oracle.attention_backward_dq_rows(qn, kn, vn, don, w.scale, causal, 0, h, rows))
        check_grad(np.stack(got), np.stack(ref), f"{name} dq rows causal={causal}",
                   row_axis=1, head_axes=(0,), rows="sampled")
        for h in (0, w.H - 1):
            hd = oracle.attention_head(qn, kn, vn, don, w.scale, causal, 0, h)
            check_grad(dk[0, :, h], hd["dk"], f"{name} dk h{h} causal={causal}", row_axis=0)
            check_grad(dv[0, :, h], hd["dv"], f"{name} dv h{h} causal={causal}", row_axis=0)
            del hd


# ----------------------------------------------------------- deterministic mode
def _det_case(c, causal, scale=None, what=""):
    q, k, v, do = (c[n].cuda() for n in ("q", "k", "v", "do"))
    D = q.shape[3]
    sc = D ** -0.5 if scale is None else scale
    o, lse = run_fwd(q, k, v, causal, sc)
    dq1, dk1, dv1 = fa.backward(q, k, v, o, lse, do, causal=causal, scale=sc, deterministic=True)
    dq2, dk2, dv2 = fa.backward(q, k, v, o, lse, do, causal=causal, scale=sc, deterministic=True)
    torch.cuda.synchronize()
    st, detail = fa.fa_last_device_status()
    assert st == 0, f"device status {st} {detail}"
    for x, y, name in ((dq1, dq2, "dq"), (dk1, dk2, "dk"), (dv1, dv2, "dv")):
        assert torch.equal(x, y), f"{what}: {name} differs between two deterministic runs"
    qn, kn, vn, don = (np64(c[n]) for n in ("q", "k", "v", "do"))
    dq_r, dk_r, dv_r, _ = oracle.attention_backward(qn, kn, vn, don, sc, causal)
    for name, g, r in (("dq", dq1, dq_r), ("dk", dk1, dk_r), ("dv", dv1, dv_r)):
        check_grad(np64(g), r, f"{what} det {name}", row_axis=1, head_axes=(0, 2))
    # the atomic path sums the same fp32 blocks in another order
    dqa, dka, dva = run_bwd(q, k, v, o, lse, do, causal, sc)
    assert torch.equal(dka, dk1) and torch.equal(dva, dv1)
    assert rel_l2(np64(dqa), np64(dq1)) < 2e-3


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("S", [1, 127, 129, 640])
def test_bwd_deterministic_square(D, causal, S):
    _det_case(random_case(1, 2, S, S, D, torch.bfloat16, 4000 + S), causal, what=f"S{S} D{D} c{causal}")


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("Sq,Sk", [(100, 37), (129, 700), (700, 129), (513, 255)])
def test_bwd_deterministic_rectangular(causal, Sq, Sk):
    _det_case(random_case(2, 3, Sq, Sk, 128, torch.float16, 77 + Sq + Sk), causal, what=f"Sq{Sq} Sk{Sk}")


@pytest.mark.parametrize("D", [40, 96])
def test_bwd_deterministic_other_head_dims(D):
    _det_case(random_case(2, 2, 300, 257, D, torch.bfloat16, 500 + D), True, what=f"D{D}")


def test_bwd_deterministic_c4_full_size():
    """c4 at full size in deterministic mode: two runs bit-identical, dq close
    to the atomic path's and to the oracle on sampled rows."""
    w = WORKLOADS["c4"]
    inp = make_inputs(w)
    q, k, v, do = (inp[n].cuda() for n in ("q", "k", "v", "do"))
    o, lse = run_fwd(q, k, v, True, w.scale)
    ws = fa.workspace_for(w.B, w.H, w.S, w.D, q.device, deterministic=True)
    dq1, dk1, dv1 = fa.backward(q, k, v, o, lse, do, causal=True, scale=w.scale, workspace=ws, deterministic=True)
    dq1 = dq1.clone()
    dq2, _, _ = fa.backward(q, k, v, o, lse, do, causal=True, scale=w.scale, workspace=ws, deterministic=True)
    torch.cuda.synchronize()
    assert fa.fa_last_device_status()[0] == 0
    assert torch.equal(dq1, dq2)
    dqa, dka, dva = run_bwd(q, k, v, o, lse, do, True, w.scale)
    assert torch.equal(dka, dk1) and torch.equal(dva, dv1)
    assert rel_l2(np64(dqa), np64(dq1)) < 2e-3
    rows = sample_rows(w.S, 128, 40, w.seed)
    qn, kn, vn, don = (np64(inp[n]) for n in ("q", "k", "v", "do"))
    got = np.stack([np64(dq1)[0, rows, h] for h in (0, w.H - 1)])
    ref = np.stack([oracle.attention_backward_dq_rows(qn, kn, vn, don, w.scale, True, 0, h, rows) for h in (0, w.H - 1)])
    check_grad(got, ref, "c4 det dq rows", row_axis=1, head_axes=(0,), rows="sampled")
