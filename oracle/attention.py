"""fp64 CPU oracle for exact scaled dot-product attention, forward and backward.

TEST INFRASTRUCTURE ONLY. Nothing in the product path may import, call or run
this module: only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` use it. It shares no code with the CUDA library.

What it computes is the plain definition, written out: the pages state more
than once that the fused method is exact, not an approximation
([P1] "性能引擎", [P2] opening section, [P3] "FlashAttention 到底快在哪里？"),
so the oracle materialises the full score and probability matrices in fp64 and
does nothing clever. Matrix products use numpy's matmul as a library
primitive; there is no blocking or fusion except in
``attention_forward_online``, which restates the blockwise recurrence on
purpose so that it can be checked against the two-pass definition.

Tensors are numpy arrays (any float dtype; converted to fp64 on entry) laid
out [B, S, H, D] like the library; the logsumexp is [B, H, Sq].

Conventions (readings where the pages are silent or garbled):

* scale: taken as an argument; the workloads use 1/sqrt(D) ([P1] "性能引擎"
  formula softmax(QK^T / sqrt(d_k)) V).
* logsumexp: natural log of the scaled scores, LSE_i = ln sum_j exp(scale *
  q_i . k_j) over allowed keys ([P4] §3.1 says only "logsumexp").
* causal mask with Sq != Sk: bottom-right aligned, key j allowed for query i
  iff j <= i + (Sk - Sq); with Sq == Sk this is the usual lower triangle
  ([P1] "实战集成" and [P4] §4 name only "causal"). A query row with no
  allowed key gets O = 0 and LSE = -inf.
* backward: the textbook gradient of softmax(x) V (the pages only say that the
  backward recomputes the forward, [P1] "性能引擎", [P2] item 3 "重计算",
  and that it takes five matrix products, [P4] §3.3).

Page legend: [P1] "Miniconda-Python3.9环境下使用FlashAttention优化训练";
[P2] "使用FlashAttention优化PyTorch模型注意力计算"; [P3]
"FlashAttention集成进展：PyTorch-CUDA-v2.7能否自动启用？"; [P4] the
FlashAttention-2 walkthrough published under the title "企业官网建设流程全解析";
[P5] the FlashAttention "IO感知" overview (0539edu.com/news/165270).

Every function here is pinned by ``tests/test_oracle_pins.py``.
"""
from __future__ import annotations

import numpy as np


def _f64(x):
    return np.asarray(x, dtype=np.float64)


def _bh(x):
    """[B, S, H, D] -> [B, H, S, D] fp64 view, so that matmul runs per (b, h)."""
    return _f64(x).transpose(0, 2, 1, 3)


def _bs(x):
    """[B, H, S, D] -> [B, S, H, D]."""
    return x.transpose(0, 2, 1, 3)


def allowed_mask(Sq: int, Sk: int, causal: bool) -> np.ndarray:
    """Boolean [Sq, Sk]: True where query i may attend to key j.

    Causal: bottom-right aligned, j <= i + (Sk - Sq) (reading stated in the
    module docstring). Non-causal: all True.
    """
    if not causal:
        return np.ones((Sq, Sk), dtype=bool)
    i = np.arange(Sq)[:, None]
    j = np.arange(Sk)[None, :]
    return j <= i + (Sk - Sq)


def scaled_scores(q, k, scale: float, causal: bool) -> np.ndarray:
    """x = scale * Q K^T per (b, h), masked entries set to -inf. [B, H, Sq, Sk].

    The first of the three steps of standard attention ([P1] "性能引擎":
    S = QK^T, then softmax, then multiply by V).
    """
    x = scale * (_bh(q) @ _bh(k).swapaxes(-1, -2))
    m = allowed_mask(q.shape[1], k.shape[1], causal)
    return np.where(m[None, None], x, -np.inf)


def _row_logsumexp(x: np.ndarray) -> np.ndarray:
    """ln sum_j exp(x_ij) along the last axis; -inf for rows that are all -inf."""
    m = np.max(x, axis=-1, keepdims=True)
    m_safe = np.where(np.isfinite(m), m, 0.0)
    s = np.sum(np.exp(x - m_safe), axis=-1, keepdims=True)
    with np.errstate(divide="ignore"):
        out = m_safe + np.log(s)
    return out[..., 0]


def attention_probs(q, k, scale: float, causal: bool):
    """P = softmax(scale * Q K^T [+ mask]) and the row logsumexp.

    Returns (P [B, H, Sq, Sk], LSE [B, H, Sq]). Rows with no allowed key are
    all zero in P and -inf in LSE.
    """
    x = scaled_scores(q, k, scale, causal)
    lse = _row_logsumexp(x)
    lse_safe = np.where(np.isfinite(lse), lse, 0.0)
    p = np.exp(x - lse_safe[..., None])  # exp(-inf) = 0 on masked entries
    return p, lse


def attention_forward(q, k, v, scale: float, causal: bool):
    """Two-pass definition: O = softmax(scale Q K^T [+ mask]) V, and LSE.

    q [B,Sq,H,D], k/v [B,Sk,H,D] -> (O [B,Sq,H,D], LSE [B,H,Sq]).
    ([P1] "性能引擎" formula; [P2] "实战代码对比" einsum restatement.)
    """
    p, lse = attention_probs(q, k, scale, causal)
    o = _bs(p @ _bh(v))
    return o, lse


def attention_forward_online(q, k, v, scale: float, causal: bool, block_sizes):
    """Blockwise forward with a running row max m and running sum l.

    Follows the recurrence of [P2] item 2 "分块处理" (for each K/V block:
    partial QK^T, update m and the normaliser with an online softmax,
    accumulate the output) in the unscaled-output form of [P4] §3.1: the
    accumulator is kept unscaled and divided by l once at the end, and only the
    logsumexp is kept. The printed update on [P4] §3.1 is garbled (it
    multiplies the old output by diag(l_old)); the reading used is
        m_new = max(m_old, rowmax(X_blk))
        O~    = diag(exp(m_old - m_new)) O~ + exp(X_blk - m_new) V_blk
        l     = exp(m_old - m_new) l + rowsum(exp(X_blk - m_new))
        O     = diag(l)^-1 O~,   LSE = m + ln l
    which is the only form that is exact with an unscaled O~.

    ``block_sizes`` is a list of K/V block lengths that sums to Sk.
    """
    q, k, v = _bh(q), _bh(k), _bh(v)
    B, H, Sq, D = q.shape
    Sk = k.shape[2]
    if sum(block_sizes) != Sk or any(b <= 0 for b in block_sizes):
        raise ValueError("block_sizes must be positive and sum to Sk")
    allowed = allowed_mask(Sq, Sk, causal)
    o_acc = np.zeros((B, H, Sq, v.shape[3]))
    m = np.full((B, H, Sq), -np.inf)
    l = np.zeros((B, H, Sq))
    start = 0
    for n in block_sizes:
        kb, vb = k[:, :, start:start + n], v[:, :, start:start + n]
        x = scale * (q @ kb.swapaxes(-1, -2))
        x = np.where(allowed[None, None, :, start:start + n], x, -np.inf)
        m_new = np.maximum(m, np.max(x, axis=-1))
        m_use = np.where(np.isfinite(m_new), m_new, 0.0)
        alpha = np.exp(m - m_use)              # 0 when m was -inf
        p = np.exp(x - m_use[..., None])       # 0 on masked entries
        o_acc = alpha[..., None] * o_acc + p @ vb
        l = alpha * l + np.sum(p, axis=-1)
        m = m_new
        start += n
    with np.errstate(divide="ignore", invalid="ignore"):
        o = np.where(l[..., None] > 0, o_acc / np.where(l > 0, l, 1.0)[..., None], 0.0)
        lse = np.where(l > 0, m + np.log(np.where(l > 0, l, 1.0)), -np.inf)
    return _bs(o), lse


def delta_rowsum(o, do) -> np.ndarray:
    """Dvec_i = sum_d dO_id * O_id per (b, h, i): [B, H, Sq].

    Equal to sum_j P_ij dP_ij (the row term of the softmax gradient), which is
    what lets the backward avoid a second pass over the keys.
    """
    return np.einsum("bihd,bihd->bhi", _f64(o), _f64(do))


def attention_backward(q, k, v, do, scale: float, causal: bool):
    """Gradients of L = sum(dO * O) for O = attention_forward(q, k, v).

    With P = softmax(X), X = scale Q K^T (+ mask):
        dV = P^T dO
        dP = dO V^T
        Dvec_i = sum_j P_ij dP_ij
        dX = P * (dP - Dvec)
        dQ = scale dX K,   dK = scale dX^T Q
    Five matrix products, as [P4] §3.3 counts for the backward. Returns
    (dq [B,Sq,H,D], dk [B,Sk,H,D], dv [B,Sk,H,D], dvec [B,H,Sq]).
    """
    p, _ = attention_probs(q, k, scale, causal)
    qh, kh, vh, doh = _bh(q), _bh(k), _bh(v), _bh(do)
    dv = p.swapaxes(-1, -2) @ doh
    dp = doh @ vh.swapaxes(-1, -2)
    dvec = np.sum(p * dp, axis=-1)
    dx = p * (dp - dvec[..., None])
    dq = scale * (dx @ kh)
    dk = scale * (dx.swapaxes(-1, -2) @ qh)
    return _bs(dq), _bs(dk), _bs(dv), dvec


# ---------------------------------------------------------------------------
# Row-sampled and per-head forms for workloads too large to materialise whole.
# They restate the same definitions on a subset; the tests check that they
# agree with the full forms on small inputs.
# ---------------------------------------------------------------------------

def _rows_scores(q, k, scale, causal, b, h, rows):
    rows = np.asarray(rows, dtype=np.int64)
    Sq, Sk = q.shape[1], k.shape[1]
    x = scale * (_f64(q[b, rows, h]) @ _f64(k[b, :, h]).T)        # [R, Sk]
    if causal:
        j = np.arange(Sk)[None, :]
        x = np.where(j <= rows[:, None] + (Sk - Sq), x, -np.inf)
    return x


def attention_forward_rows(q, k, v, scale, causal, b, h, rows):
    """O[b, rows, h, :] and LSE[b, h, rows] by the two-pass definition."""
    x = _rows_scores(q, k, scale, causal, b, h, rows)
    lse = _row_logsumexp(x)
    lse_safe = np.where(np.isfinite(lse), lse, 0.0)
    p = np.exp(x - lse_safe[:, None])
    return p @ _f64(v[b, :, h]), lse


def attention_backward_dq_rows(q, k, v, do, scale, causal, b, h, rows):
    """dQ[b, rows, h, :]: row i needs only its own P_i., dP_i. and Dvec_i."""
    x = _rows_scores(q, k, scale, causal, b, h, rows)
    lse = _row_logsumexp(x)
    lse_safe = np.where(np.isfinite(lse), lse, 0.0)
    p = np.exp(x - lse_safe[:, None])                              # [R, Sk]
    dp = _f64(do[b, rows, h]) @ _f64(v[b, :, h]).T                 # [R, Sk]
    dvec = np.sum(p * dp, axis=-1, keepdims=True)
    return scale * ((p * (dp - dvec)) @ _f64(k[b, :, h]))


def attention_head(q, k, v, do, scale, causal, b, h):
    """Full forward and backward of one (b, h) head.

    Returns dict with o [Sq,D], lse [Sq], dq [Sq,D], dk [Sk,D], dv [Sk,D].
    """
    sl = (slice(b, b + 1), slice(None), slice(h, h + 1))
    qq, kk, vv, dd = q[sl], k[sl], v[sl], do[sl]
    o, lse = attention_forward(qq, kk, vv, scale, causal)
    dq, dk, dv, _ = attention_backward(qq, kk, vv, dd, scale, causal)
    return {"o": o[0, :, 0], "lse": lse[0, 0], "dq": dq[0, :, 0],
            "dk": dk[0, :, 0], "dv": dv[0, :, 0]}
