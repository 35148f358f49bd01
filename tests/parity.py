"""Shared helpers for the GPU parity tests: run the library through its C ABI,
run the fp64 oracle on the same (rounded) inputs, and compare with the
tolerances the workloads fix: max-abs |O| error <= 1e-2 (fp16) / 2e-2 (bf16),
max-abs LSE error <= 1e-3, relative L2 error <= 5e-2 for dQ, dK and dV."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from exact_io_aware_96_b200 import fa

O_TOL = {torch.float16: 1e-2, torch.bfloat16: 2e-2}
LSE_TOL = 1e-3
GRAD_TOL = 5e-2


def np64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def to_dev(d):
    return {k: v.cuda() for k, v in d.items()}


def check_o_lse(o_gpu, lse_gpu, o_ref, lse_ref, dtype, what=""):
    o_gpu, lse_gpu = np.asarray(o_gpu, np.float64), np.asarray(lse_gpu, np.float64)
    assert np.all(np.isfinite(o_gpu)), f"{what}: non-finite O"
    err = np.max(np.abs(o_gpu - o_ref)) if o_ref.size else 0.0
    assert err <= O_TOL[dtype], f"{what}: O max-abs error {err:.3e} > {O_TOL[dtype]}"
    fin = np.isfinite(lse_ref)
    assert np.array_equal(fin, np.isfinite(lse_gpu)), f"{what}: LSE finiteness differs"
    assert np.all(lse_gpu[~fin] == -np.inf), f"{what}: masked rows must have LSE = -inf"
    if fin.any():
        lerr = np.max(np.abs(lse_gpu[fin] - lse_ref[fin]))
        assert lerr <= LSE_TOL, f"{what}: LSE max-abs error {lerr:.3e} > {LSE_TOL}"
    return err


def rel_l2(a, b):
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    nb = np.linalg.norm(b)
    return np.linalg.norm(a - b) / (nb if nb > 0 else 1.0)


def check_grad(g_gpu, g_ref, what=""):
    g_gpu = np.asarray(g_gpu, np.float64)
    assert np.all(np.isfinite(g_gpu)), f"{what}: non-finite gradient"
    e = rel_l2(g_gpu, g_ref)
    assert e <= GRAD_TOL, f"{what}: relative L2 error {e:.3e} > {GRAD_TOL}"
    return e


def run_fwd(q, k, v, causal, scale=None):
    o, lse = fa.forward(q, k, v, causal=causal, scale=scale)
    torch.cuda.synchronize()
    st, detail = fa.fa_last_device_status()
    assert st == 0, f"device status {st} {detail}"
    return o, lse


def run_bwd(q, k, v, o, lse, do, causal, scale=None):
    dq, dk, dv = fa.backward(q, k, v, o, lse, do, causal=causal, scale=scale)
    torch.cuda.synchronize()
    st, detail = fa.fa_last_device_status()
    assert st == 0, f"device status {st} {detail}"
    return dq, dk, dv


def full_check(inp_cpu, causal, scale=None, backward=True, what=""):
    """Whole-tensor parity of forward (and backward) against the oracle."""
    q, k, v, do = (inp_cpu[n] for n in ("q", "k", "v", "do"))
    dtype = q.dtype
    D = q.shape[3]
    sc = D ** -0.5 if scale is None else scale
    dev = {n: inp_cpu[n].cuda() for n in ("q", "k", "v", "do")}
    o, lse = run_fwd(dev["q"], dev["k"], dev["v"], causal, sc)
    o_ref, lse_ref = oracle.attention_forward(np64(q), np64(k), np64(v), sc, causal)
    check_o_lse(np64(o), np64(lse), o_ref, lse_ref, dtype, what + " fwd")
    if not backward:
        return
    dq, dk, dv = run_bwd(dev["q"], dev["k"], dev["v"], o, lse, dev["do"], causal, sc)
    dq_r, dk_r, dv_r, _ = oracle.attention_backward(np64(q), np64(k), np64(v), np64(do), sc, causal)
    for name, g, r in (("dq", dq, dq_r), ("dk", dk, dk_r), ("dv", dv, dv_r)):
        check_grad(np64(g), r, f"{what} {name}")
