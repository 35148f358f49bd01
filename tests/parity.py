"""Shared helpers for the GPU parity tests: run the library through its C ABI,
run the fp64 oracle on the same (rounded) inputs, and compare with the
tolerances the workloads fix: max-abs |O| error <= 1e-2 (fp16) / 2e-2 (bf16),
max-abs LSE error <= 1e-3, relative L2 error <= 5e-2 for dQ, dK and dV."""
from __future__ import annotations

import numpy as np
import torch

import oracle
import oracle.fp8
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


def blocks_rel_l2(a, b, row_axis, head_axes=(), block=128, rows=None, floor=1e-3):
    """Relative L2 error of every (head, 128-row block) piece of ``a`` against
    ``b``: ||a_p - b_p|| / max(||b_p||, f_p), where f_p = floor * ||b|| *
    sqrt(size_p / size) is a small fraction of the piece's share of the whole
    norm (it only matters for pieces whose reference is, by cancellation,
    almost zero). ``rows`` gives the sequence index of each position along
    ``row_axis`` (default 0, 1, ...; sampled rows are grouped by the block
    they fall in). Yields ((head indices, first row of the block), error)."""
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    nb_all = np.linalg.norm(b)
    n = a.shape[row_axis]
    blk = (np.arange(n) if rows is None else np.asarray(rows)) // block
    heads = [a.shape[ax] for ax in head_axes]
    for idx in np.ndindex(*heads):
        for kb in np.unique(blk):
            sl = [slice(None)] * a.ndim
            sl[row_axis] = np.nonzero(blk == kb)[0]
            for ax, i in zip(head_axes, idx):
                sl[ax] = i
            pa, pb = a[tuple(sl)], b[tuple(sl)]
            share = nb_all * np.sqrt(pb.size / b.size) if b.size else 0.0
            den = max(np.linalg.norm(pb), floor * share)
            err = np.linalg.norm(pa - pb) / den if den > 0 else np.linalg.norm(pa - pb)
            yield (idx, int(kb) * block), float(err)


def check_grad(g_gpu, g_ref, what="", row_axis=None, head_axes=(), rows=None):
    """Relative L2 error <= GRAD_TOL over the whole tensor and, when
    ``row_axis`` is given, over every head and every 128-row block along that
    axis (the same bar applied piece by piece, so that an error confined to
    one block or one head cannot hide in the norm of the rest).

    ``rows="sampled"``: the positions along ``row_axis`` are a sample of rows,
    and the pieces are whole heads. A block holds only one to three sampled
    rows, and a single row's gradient can be small by cancellation (a row whose
    attention sits on one key has dP - Dvec close to 0), where the fixed
    rounding of dP and Dvec is a large fraction of it."""
    if isinstance(rows, str) and rows == "sampled":
        rows = np.zeros(np.asarray(g_gpu).shape[row_axis], dtype=np.int64)
    g_gpu = np.asarray(g_gpu, np.float64)
    assert np.all(np.isfinite(g_gpu)), f"{what}: non-finite gradient"
    e = rel_l2(g_gpu, g_ref)
    assert e <= GRAD_TOL, f"{what}: relative L2 error {e:.3e} > {GRAD_TOL}"
    if row_axis is not None:
        worst = max(blocks_rel_l2(g_gpu, g_ref, row_axis, head_axes, rows=rows), key=lambda x: x[1])
        assert worst[1] <= GRAD_TOL, (f"{what}: relative L2 error {worst[1]:.3e} > {GRAD_TOL} in the piece "
                                      f"(head index {worst[0][0]}, rows from {worst[0][1]})")
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
        check_grad(np64(g), r, f"{what} {name}", row_axis=1, head_axes=(0, 2))


# ------------------------------------------------------------------ e4m3 forward
# Half a unit in the last place of the output type, relative: bf16 keeps 8
# significant bits, fp16 11.
OUT_HALF_ULP = {torch.bfloat16: 2.0 ** -8, torch.float16: 2.0 ** -11}


def run_fwd_fp8(q8, k8, v8, qd, kd, vd, causal, scale=None, out_dtype=torch.bfloat16):
    o, lse = fa.forward_fp8(q8, k8, v8, qd, kd, vd, causal=causal, scale=scale, out_dtype=out_dtype)
    torch.cuda.synchronize()
    st, detail = fa.fa_last_device_status()
    assert st == 0, f"device status {st} {detail}"
    return o, lse


def check_fp8_o_lse(o_gpu, lse_gpu, qn, kn, vn, scale, causal, out_dtype, b, h, rows, what=""):
    """O[b, rows, h] and LSE[b, h, rows] of the e4m3 forward against exact
    attention on the dequantized inputs (qn, kn, vn fp64).

    The kernel differs from exact attention by (1) rounding P to E4M3 before
    the P V product, (2) the rounding of O to ``out_dtype``, (3) fp32
    arithmetic and exp2 approximations (relative 2^-13 at most, below 2^-8 of
    (1)). Two bars:
    * every element within the worst case of (1) from
      ``oracle.fp8.e4m3_p_rounding_bound`` (times 1 + 2^-8 for (3)), plus
      (2), half an ulp of |O|;
    * when at least 2048 elements are compared, the summed squared error
      within twice the expected value of (1) + (2) (the oracle's variance bound
      plus u^2 |O|^2 / 3), a bar that a wrong key, row or column breaks.
    LSE does not see the rounding of P (the row sum uses the unrounded values):
    the 16-bit path's bar applies.
    """
    o_gpu, lse_gpu = np.asarray(o_gpu, np.float64), np.asarray(lse_gpu, np.float64)
    assert np.all(np.isfinite(o_gpu)), f"{what}: non-finite O"
    o_ref, lse_ref = oracle.attention_forward_rows(qn, kn, vn, scale, causal, b, h, rows)
    fin = np.isfinite(lse_ref)
    assert np.array_equal(fin, np.isfinite(lse_gpu)), f"{what}: LSE finiteness differs"
    assert np.all(lse_gpu[~fin] == -np.inf), f"{what}: masked rows must have LSE = -inf"
    if fin.any():
        lerr = np.max(np.abs(lse_gpu[fin] - lse_ref[fin]))
        assert lerr <= LSE_TOL, f"{what}: LSE max-abs error {lerr:.3e} > {LSE_TOL}"
    u = OUT_HALF_ULP[out_dtype]
    bound = oracle.fp8.e4m3_p_rounding_bound(qn, kn, vn, scale, causal, b, h, rows)
    tol = bound * (1 + 2.0 ** -8) + u * (np.abs(o_ref) + bound) + 1e-6
    err = np.abs(o_gpu - o_ref)
    bad = err > tol
    assert not bad.any(), (f"{what}: {bad.sum()} elements beyond the e4m3 bound; worst err "
                           f"{err[bad].max():.3e} vs tol {tol[bad][np.argmax(err[bad])]:.3e}")
    if err.size >= 2048:
        var = oracle.fp8.e4m3_p_rounding_variance(qn, kn, vn, scale, causal, b, h, rows)
        expect = var.sum() + (u * u / 3.0) * np.sum(o_ref ** 2)
        e2 = np.sum(err ** 2)
        assert e2 <= 2.0 * expect + 1e-12, f"{what}: squared error {e2:.3e} > 2 x expected {expect:.3e}"
    return float(err.max()) if err.size else 0.0
