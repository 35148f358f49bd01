"""Checks that pin the fp64 oracle to facts fixed outside itself.

Each ``check_*`` takes an oracle module (the real one, or a copy with a
planted mistake in ``test_oracle_mutants.py``) and raises AssertionError when
the oracle disagrees with a hand-derived closed form, a mathematical
invariant, a brute-force computation, a numerical derivative or an
independent library routine (torch's scaled_dot_product_attention in fp64).
"""
from __future__ import annotations

import json
import math
import os

import numpy as np
import torch
import torch.nn.functional as F

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "worked_examples.json")


def _rand(rng, *shape, std=1.0):
    return rng.standard_normal(shape) * std


def _case(rng, B, H, Sq, Sk, D, std=1.0):
    q = _rand(rng, B, Sq, H, D, std=std)
    k = _rand(rng, B, Sk, H, D, std=std)
    v = _rand(rng, B, Sk, H, D)
    do = _rand(rng, B, Sq, H, D)
    return q, k, v, do


SHAPES = [  # (B, H, Sq, Sk, D)
    (1, 1, 1, 1, 1), (1, 1, 5, 5, 3), (2, 3, 7, 7, 4), (1, 2, 4, 9, 8),
    (1, 1, 9, 4, 2), (2, 1, 16, 16, 8), (1, 2, 3, 11, 5),
]


def _ev(expr):
    return float(eval(expr, {"__builtins__": {}}, {"e": math.e, "log": math.log, "exp": math.exp}))


def check_golden(orc):
    """Hand-worked closed forms (tests/golden/worked_examples.json)."""
    data = json.load(open(GOLDEN))
    for ex in data["examples"]:
        q = np.array(ex["q"], dtype=np.float64)[None, :, None, :]
        k = np.array(ex["k"], dtype=np.float64)[None, :, None, :]
        v = np.array(ex["v"], dtype=np.float64)[None, :, None, :]
        scale = _ev(ex["scale"])
        for key, causal in (("noncausal", False), ("causal", True)):
            o, lse = orc.attention_forward(q, k, v, scale, causal)
            want_o = np.array([[_ev(x) for x in row] for row in ex[key]["o"]])
            want_l = np.array([_ev(x) for x in ex[key]["lse"]])
            assert np.allclose(o[0, :, 0], want_o, rtol=0, atol=1e-14), (ex["name"], key, o[0, :, 0], want_o)
            assert np.allclose(lse[0, 0], want_l, rtol=0, atol=1e-14), (ex["name"], key, lse[0, 0], want_l)


def check_online_equals_two_pass(orc, seed=0):
    """Blockwise recurrence == two-pass definition, random block splits."""
    rng = np.random.default_rng(seed)
    for (B, H, Sq, Sk, D) in SHAPES:
        q, k, v, _ = _case(rng, B, H, Sq, Sk, D, std=2.0)
        for causal in (False, True):
            o2, l2 = orc.attention_forward(q, k, v, 0.7, causal)
            for _ in range(3):
                sizes, left = [], Sk
                while left:
                    n = int(rng.integers(1, left + 1))
                    sizes.append(n)
                    left -= n
                o1, l1 = orc.attention_forward_online(q, k, v, 0.7, causal, sizes)
                fin = np.isfinite(l2)
                assert np.array_equal(fin, np.isfinite(l1))
                assert np.max(np.abs(o1 - o2)) <= 1e-12
                assert np.max(np.abs(l1[fin] - l2[fin])) <= 1e-12


def check_probability_rows(orc, seed=1):
    """P >= 0, rows sum to 1 over allowed keys, masked entries are exactly 0."""
    rng = np.random.default_rng(seed)
    for (B, H, Sq, Sk, D) in SHAPES:
        q, k, _, _ = _case(rng, B, H, Sq, Sk, D, std=3.0)
        for causal in (False, True):
            p, lse = orc.attention_probs(q, k, 0.5, causal)
            assert np.all(p >= 0)
            i = np.arange(Sq)[:, None]
            j = np.arange(Sk)[None, :]
            allowed = (j <= i + (Sk - Sq)) if causal else np.ones((Sq, Sk), bool)
            assert np.all(p[..., ~allowed] == 0)
            has = allowed.any(axis=1)
            s = p.sum(-1)
            assert np.allclose(s[..., has], 1.0, atol=1e-13)
            assert np.all(s[..., ~has] == 0)
            assert np.all(np.isneginf(lse[..., ~has]))


def check_zero_query(orc, seed=2):
    """Q = 0: every allowed key has equal weight.
    Non-causal O_i = mean_j V_j, LSE_i = ln Sk; causal (Sq == Sk) O_i = mean_{j<=i} V_j, LSE_i = ln(i+1)."""
    rng = np.random.default_rng(seed)
    for (B, H, S, D) in ((1, 1, 6, 3), (2, 2, 9, 4)):
        _, k, v, _ = _case(rng, B, H, S, S, D)
        q = np.zeros((B, S, H, D))
        o, lse = orc.attention_forward(q, k, v, 0.3, False)
        assert np.allclose(o, np.broadcast_to(v.mean(axis=1, keepdims=True), o.shape), atol=1e-14)
        assert np.allclose(lse, math.log(S), atol=1e-14)
        o, lse = orc.attention_forward(q, k, v, 0.3, True)
        prefix = np.cumsum(v, axis=1) / np.arange(1, S + 1)[None, :, None, None]
        assert np.allclose(o, prefix, atol=1e-13)
        assert np.allclose(lse, np.log(np.arange(1, S + 1))[None, None, :], atol=1e-14)


def check_causal_row0(orc, seed=3):
    """Causal (Sq == Sk): row 0 sees only key 0, so O_0 = V_0 and LSE_0 = scale q_0 . k_0."""
    rng = np.random.default_rng(seed)
    q, k, v, _ = _case(rng, 2, 3, 7, 7, 5)
    o, lse = orc.attention_forward(q, k, v, 0.45, True)
    assert np.allclose(o[:, 0], v[:, 0], atol=1e-14)
    want = 0.45 * np.einsum("bhd,bhd->bh", q[:, 0], k[:, 0])
    assert np.allclose(lse[:, :, 0], want, atol=1e-13)


def check_key_permutation(orc, seed=4):
    """Non-causal: permuting K and V rows together leaves O, LSE and dQ unchanged and
    permutes dK and dV the same way."""
    rng = np.random.default_rng(seed)
    q, k, v, do = _case(rng, 1, 2, 6, 8, 4)
    perm = rng.permutation(8)
    o1, l1 = orc.attention_forward(q, k, v, 0.6, False)
    o2, l2 = orc.attention_forward(q, k[:, perm], v[:, perm], 0.6, False)
    assert np.allclose(o1, o2, atol=1e-13) and np.allclose(l1, l2, atol=1e-13)
    g1 = orc.attention_backward(q, k, v, do, 0.6, False)
    g2 = orc.attention_backward(q, k[:, perm], v[:, perm], do, 0.6, False)
    assert np.allclose(g1[0], g2[0], atol=1e-13)
    assert np.allclose(g1[1][:, perm], g2[1], atol=1e-13)
    assert np.allclose(g1[2][:, perm], g2[2], atol=1e-13)


def check_constant_values(orc, seed=5):
    """V = c (every row the same vector): O = c, and O does not depend on Q or K,
    so dQ = dK = 0; dV_j = sum_i P_ij dO_i sums to sum_i dO_i over j."""
    rng = np.random.default_rng(seed)
    for causal in (False, True):
        q, k, _, do = _case(rng, 1, 2, 5, 5, 3)
        c = rng.standard_normal(3)
        v = np.broadcast_to(c, (1, 5, 2, 3)).copy()
        o, _ = orc.attention_forward(q, k, v, 0.8, causal)
        assert np.allclose(o, np.broadcast_to(c, o.shape), atol=1e-14)
        dq, dk, dv, _ = orc.attention_backward(q, k, v, do, 0.8, causal)
        assert np.max(np.abs(dq)) <= 1e-13 and np.max(np.abs(dk)) <= 1e-13
        assert np.allclose(dv.sum(axis=1), do.sum(axis=1), atol=1e-13)


def check_single_key(orc, seed=6):
    """Sk = 1: P = 1 for every query, so O_i = V_0, LSE_i = scale q_i . k_0,
    dV_0 = sum_i dO_i and dQ = dK = 0."""
    rng = np.random.default_rng(seed)
    q, k, v, do = _case(rng, 1, 1, 4, 1, 3)
    o, lse = orc.attention_forward(q, k, v, 0.9, False)
    assert np.allclose(o, np.broadcast_to(v[:, :1], o.shape), atol=1e-14)
    assert np.allclose(lse[0, 0], 0.9 * q[0, :, 0] @ k[0, 0, 0], atol=1e-14)
    dq, dk, dv, _ = orc.attention_backward(q, k, v, do, 0.9, False)
    assert np.max(np.abs(dq)) <= 1e-14 and np.max(np.abs(dk)) <= 1e-14
    assert np.allclose(dv[0, 0, 0], do[0, :, 0].sum(axis=0), atol=1e-14)


def check_bounds(orc, seed=7):
    """Each O_i lies in the per-column hull of the allowed V rows, and
    max_j x_ij <= LSE_i <= max_j x_ij + ln(#allowed keys)."""
    rng = np.random.default_rng(seed)
    q, k, v, _ = _case(rng, 1, 2, 8, 8, 4, std=2.0)
    for causal in (False, True):
        o, lse = orc.attention_forward(q, k, v, 0.5, causal)
        x = 0.5 * np.einsum("bihd,bjhd->bhij", q, k)
        for i in range(8):
            n = i + 1 if causal else 8
            xm = x[..., i, :n].max(-1)
            assert np.all(lse[..., i] >= xm - 1e-13)
            assert np.all(lse[..., i] <= xm + math.log(n) + 1e-13)
            lo = v[:, :n].min(axis=1)
            hi = v[:, :n].max(axis=1)
            assert np.all(o[:, i] >= lo - 1e-13) and np.all(o[:, i] <= hi + 1e-13)


def check_finite_differences(orc, seed=8):
    """Central differences of L = sum(dO * O) match the analytic gradients."""
    rng = np.random.default_rng(seed)
    h = 1e-6
    for (Sq, Sk, D, causal) in ((5, 5, 3, False), (5, 5, 3, True), (3, 6, 4, True), (6, 4, 2, False), (8, 8, 8, True)):
        q, k, v, do = _case(rng, 1, 1, Sq, Sk, D)
        scale = 0.7

        def loss(qq, kk, vv):
            o, _ = orc.attention_forward(qq, kk, vv, scale, causal)
            return float(np.sum(o * do))

        dq, dk, dv, _ = orc.attention_backward(q, k, v, do, scale, causal)
        for which, g in ((0, dq), (1, dk), (2, dv)):
            args = [q, k, v]
            num = np.zeros_like(args[which])
            it = np.nditer(args[which], flags=["multi_index"])
            for _ in it:
                idx = it.multi_index
                plus = [a.copy() for a in args]
                minus = [a.copy() for a in args]
                plus[which][idx] += h
                minus[which][idx] -= h
                num[idx] = (loss(*plus) - loss(*minus)) / (2 * h)
            err = np.linalg.norm(num - g) / max(np.linalg.norm(g), 1e-30)
            assert err <= 1e-6, (Sq, Sk, D, causal, which, err)


def _torch_ref(q, k, v, do, scale, causal):
    """torch's SDPA (math path on CPU) in fp64, [B,S,H,D] in and out, with autograd."""
    t = [torch.tensor(a.transpose(0, 2, 1, 3), dtype=torch.float64, requires_grad=True) for a in (q, k, v)]
    Sq, Sk = q.shape[1], k.shape[1]
    mask = None
    if causal:
        i = torch.arange(Sq)[:, None]
        j = torch.arange(Sk)[None, :]
        mask = j <= i + (Sk - Sq)
    o = F.scaled_dot_product_attention(t[0], t[1], t[2], attn_mask=mask, scale=scale)
    o.backward(torch.tensor(do.transpose(0, 2, 1, 3)))
    to = lambda x: x.detach().numpy().transpose(0, 2, 1, 3)
    return to(o), to(t[0].grad), to(t[1].grad), to(t[2].grad)


def check_torch_sdpa(orc, seed=9):
    """Independent library routine: torch.nn.functional.scaled_dot_product_attention
    in fp64 on the CPU, forward and autograd backward."""
    rng = np.random.default_rng(seed)
    for (B, H, Sq, Sk, D) in ((2, 3, 7, 7, 4), (1, 2, 5, 9, 8), (1, 1, 16, 16, 16), (2, 2, 33, 20, 8)):
        q, k, v, do = _case(rng, B, H, Sq, Sk, D, std=1.5)
        for causal in (False, True):
            if causal and Sq > Sk:
                continue  # rows with no allowed key: torch returns NaN there
            o_t, dq_t, dk_t, dv_t = _torch_ref(q, k, v, do, 0.37, causal)
            o, _ = orc.attention_forward(q, k, v, 0.37, causal)
            dq, dk, dv, _ = orc.attention_backward(q, k, v, do, 0.37, causal)
            for a, b in ((o, o_t), (dq, dq_t), (dk, dk_t), (dv, dv_t)):
                assert np.max(np.abs(a - b)) <= 1e-12


def check_delta_identity(orc, seed=10):
    """sum_d dO_id O_id == sum_j P_ij dP_ij (the backward's row term)."""
    rng = np.random.default_rng(seed)
    for causal in (False, True):
        q, k, v, do = _case(rng, 2, 2, 9, 9, 4)
        o, _ = orc.attention_forward(q, k, v, 0.5, causal)
        _, _, _, dvec = orc.attention_backward(q, k, v, do, 0.5, causal)
        assert np.allclose(orc.delta_rowsum(o, do), dvec, atol=1e-13)


def check_fully_masked_rows(orc, seed=11):
    """Causal with Sq > Sk: rows i < Sq - Sk have no allowed key -> O = 0,
    LSE = -inf, and they contribute nothing to any gradient."""
    rng = np.random.default_rng(seed)
    q, k, v, do = _case(rng, 1, 2, 7, 3, 4)
    o, lse = orc.attention_forward(q, k, v, 0.5, True)
    assert np.all(o[:, :4] == 0) and np.all(np.isneginf(lse[..., :4]))
    assert np.all(np.isfinite(lse[..., 4:]))
    dq, dk, dv, _ = orc.attention_backward(q, k, v, do, 0.5, True)
    assert np.all(dq[:, :4] == 0)
    # dropping those rows changes neither dK nor dV
    _, dk2, dv2, _ = orc.attention_backward(q[:, 4:], k, v, do[:, 4:], 0.5, True)
    assert np.allclose(dk, dk2, atol=1e-14) and np.allclose(dv, dv2, atol=1e-14)


def check_row_forms(orc, seed=12):
    """Row-sampled and per-head forms agree with the full forms."""
    rng = np.random.default_rng(seed)
    q9, k9, v9, do9 = _case(rng, 1, 2, 9, 13, 4)   # Sq != Sk: the causal offset matters
    for b, h in ((0, 0), (0, 1)):
        o, lse = orc.attention_forward(q9, k9, v9, 0.4, True)
        dq = orc.attention_backward(q9, k9, v9, do9, 0.4, True)[0]
        o_r, l_r = orc.attention_forward_rows(q9, k9, v9, 0.4, True, b, h, [0, 4, 8])
        assert np.allclose(o_r, o[b, [0, 4, 8], h], atol=1e-14)
        assert np.allclose(l_r, lse[b, h, [0, 4, 8]], atol=1e-14)
        dq_r = orc.attention_backward_dq_rows(q9, k9, v9, do9, 0.4, True, b, h, [0, 4, 8])
        assert np.allclose(dq_r, dq[b, [0, 4, 8], h], atol=1e-14)
    q, k, v, do = _case(rng, 2, 3, 13, 13, 4)
    rows = [0, 3, 7, 12]
    for causal in (False, True):
        o, lse = orc.attention_forward(q, k, v, 0.4, causal)
        dq, dk, dv, _ = orc.attention_backward(q, k, v, do, 0.4, causal)
        for b in range(2):
            for h in range(3):
                o_r, l_r = orc.attention_forward_rows(q, k, v, 0.4, causal, b, h, rows)
                assert np.allclose(o_r, o[b, rows, h], atol=1e-14)
                assert np.allclose(l_r, lse[b, h, rows], atol=1e-14)
                dq_r = orc.attention_backward_dq_rows(q, k, v, do, 0.4, causal, b, h, rows)
                assert np.allclose(dq_r, dq[b, rows, h], atol=1e-14)
        hd = orc.attention_head(q, k, v, do, 0.4, causal, 1, 2)
        for name, ref in (("o", o[1, :, 2]), ("lse", lse[1, 2]), ("dq", dq[1, :, 2]),
                          ("dk", dk[1, :, 2]), ("dv", dv[1, :, 2])):
            assert np.allclose(hd[name], ref, atol=1e-14), name


ALL_CHECKS = [
    check_golden, check_online_equals_two_pass, check_probability_rows, check_zero_query,
    check_causal_row0, check_key_permutation, check_constant_values, check_single_key,
    check_bounds, check_finite_differences, check_torch_sdpa, check_delta_identity,
    check_fully_masked_rows, check_row_forms,
]
