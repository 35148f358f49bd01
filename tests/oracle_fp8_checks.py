"""Checks that pin the e4m3 oracle (``oracle.fp8``) to facts fixed outside it.

Each ``check_*`` takes the module (the real one, or a copy with a planted
mistake in ``test_oracle_fp8.py``) and raises AssertionError on a mismatch with
the E4M3 format's hand-derived values, torch's float8_e4m3fn decoding (an
independent library routine), torch's scaled_dot_product_attention in fp64, a
brute-force rounding of P, or an algebraic invariant.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np
import torch
import torch.nn.functional as F

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "e4m3_values.json")


def _ev(expr):
    return float(eval(expr, {"__builtins__": {}}, {"nan": math.nan}))


def _torch_decode(b):
    t = torch.as_tensor(np.asarray(b, dtype=np.uint8)).view(torch.float8_e4m3fn)
    return t.to(torch.float64).numpy()


def check_e4m3_closed_forms(f8):
    """Hand-derived values of the format definition (tests/golden/e4m3_values.json)."""
    for hexb, expr, note in json.load(open(GOLDEN))["values"]:
        got = float(f8.decode_e4m3(np.array([int(hexb, 16)]))[0])
        want = _ev(expr)
        if math.isnan(want):
            assert math.isnan(got), (hexb, note, got)
        else:
            assert got == want and math.copysign(1, got) == math.copysign(1, want), (hexb, note, got, want)


def check_e4m3_all_bytes_vs_torch(f8):
    """Every one of the 256 encodings against torch's float8_e4m3fn decoding."""
    b = np.arange(256)
    got, want = f8.decode_e4m3(b), _torch_decode(b)
    nan = np.isnan(want)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], want[~nan])
    assert np.array_equal(np.signbit(got[~nan]), np.signbit(want[~nan]))


def check_e4m3_order_and_sign(f8):
    """Bytes 0..126 decode to strictly increasing values; the sign bit negates."""
    pos = f8.decode_e4m3(np.arange(127))
    assert np.all(np.diff(pos) > 0)
    assert np.array_equal(f8.decode_e4m3(np.arange(127) | 0x80), -pos)


def _bytes(rng, *shape):
    """Random finite E4M3 bytes of moderate magnitude (|value| in [2^-6, 2^3))."""
    e = rng.integers(1, 10, size=shape)
    m = rng.integers(0, 8, size=shape)
    s = rng.integers(0, 2, size=shape)
    return (s << 7) | (e << 3) | m


def check_attention_vs_sdpa(f8, seed=20):
    """attention_forward_e4m3 against torch SDPA (fp64) on torch-decoded, descaled inputs."""
    rng = np.random.default_rng(seed)
    for (B, H, Sq, Sk, D), causal in (((1, 2, 5, 7, 4), False), ((2, 1, 6, 6, 8), True), ((1, 1, 9, 4, 3), True)):
        q8, k8, v8 = _bytes(rng, B, Sq, H, D), _bytes(rng, B, Sk, H, D), _bytes(rng, B, Sk, H, D)
        qd, kd, vd, scale = 0.25, 0.125, 3.0, 0.7
        o, lse = f8.attention_forward_e4m3(q8, k8, v8, qd, kd, vd, scale, causal)
        qt, kt, vt = (torch.from_numpy(_torch_decode(x) * d).permute(0, 2, 1, 3) for x, d in
                      ((q8, qd), (k8, kd), (v8, vd)))
        mask = None
        if causal:
            i = torch.arange(Sq)[:, None]
            j = torch.arange(Sk)[None, :]
            mask = j <= i + (Sk - Sq)
        ref = F.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask, scale=scale)
        ref = ref.permute(0, 2, 1, 3).numpy()
        rows = mask.any(-1).numpy() if causal else np.ones(Sq, bool)
        assert np.allclose(o[:, rows], ref[:, rows], rtol=0, atol=1e-12)
        x = scale * torch.einsum("bhid,bhjd->bhij", qt, kt)
        if causal:
            x = x.masked_fill(~mask, -math.inf)
        want_lse = torch.logsumexp(x, -1).numpy()
        fin = np.isfinite(want_lse)
        assert np.allclose(lse[fin], want_lse[fin], rtol=0, atol=1e-12)


def check_descale_algebra(f8, seed=21):
    """v_descale scales O linearly and leaves LSE alone; only scale * q_descale *
    k_descale enters the scores."""
    rng = np.random.default_rng(seed)
    q8, k8, v8 = _bytes(rng, 1, 6, 2, 8), _bytes(rng, 1, 9, 2, 8), _bytes(rng, 1, 9, 2, 8)
    o1, l1 = f8.attention_forward_e4m3(q8, k8, v8, 0.5, 0.25, 1.0, 0.3, False)
    o2, l2 = f8.attention_forward_e4m3(q8, k8, v8, 0.5, 0.25, 5.0, 0.3, False)
    assert np.allclose(o2, 5.0 * o1, rtol=1e-13, atol=0) and np.array_equal(l1, l2)
    o3, l3 = f8.attention_forward_e4m3(q8, k8, v8, 1.0, 0.5, 1.0, 0.3 * 0.25, False)
    assert np.allclose(o3, o1, rtol=1e-12, atol=1e-14) and np.allclose(l3, l1, rtol=1e-12, atol=1e-14)
    o4, _ = f8.attention_forward_e4m3(q8, k8, v8, 0.5, 0.25, 1.0, 0.3 * 3, False)
    assert not np.allclose(o4, o1)


def _round_e4m3_bruteforce(x, table_vals, table_bytes):
    """Nearest finite E4M3 value to each x >= 0 by exhaustive search; a tie goes
    to the encoding with an even mantissa (round to nearest even)."""
    d = np.abs(x[..., None] - table_vals)
    best = d.min(-1, keepdims=True)
    cand = d <= best
    even = (table_bytes & 1) == 0
    pick = np.where(cand & even, 1, 0) + np.where(cand, 1, 0)  # prefer tied even encodings
    return table_vals[np.argmax(pick, axis=-1)]


def check_p_rounding_bound(f8, seed=22):
    """Rounding every P' = c P (c >= 1) to E4M3 by brute force never moves O by
    more than e4m3_p_rounding_bound, and two built cases reach the bound."""
    bts = np.arange(127)
    vals = _torch_decode(bts)           # the rounding table comes from torch, not from the oracle
    rng = np.random.default_rng(seed)
    for trial in range(6):
        Sq, Sk, D = 5, 40, 3
        q = rng.standard_normal((1, Sq, 1, D)) * 2.0
        k = rng.standard_normal((1, Sk, 1, D)) * 2.0
        v = rng.standard_normal((1, Sk, 1, D))
        scale, causal = 0.9, trial % 2 == 1
        rows = np.arange(Sq)
        bound = f8.e4m3_p_rounding_bound(q, k, v, scale, causal, 0, 0, rows)
        x = scale * (q[0, :, 0] @ k[0, :, 0].T)
        if causal:
            x = np.where(np.arange(Sk)[None, :] <= np.arange(Sq)[:, None] + (Sk - Sq), x, -np.inf)
        p = np.exp(x - x.max(-1, keepdims=True))
        l = p.sum(-1, keepdims=True)
        o = (p @ v[0, :, 0]) / l
        for c in (1.0, 2.0 ** rng.uniform(0, 8)):
            pr = _round_e4m3_bruteforce(c * p, vals, bts) / c
            err = np.abs((pr @ v[0, :, 0]) / l - o)
            assert np.all(err <= bound * (1 + 1e-12) + 1e-15), (trial, c, (err / bound).max())
    # Built cases: two keys, P = (1, P2), V = (0, 1): only P2's rounding shows.
    for p2, want_frac in ((0.53125, 1 / 1.0625), (1.5 * 2.0 ** -9, 1.0)):
        k = np.array([0.0, math.log(p2)])[None, :, None, None]
        q = np.ones((1, 1, 1, 1))
        v = np.array([0.0, 1.0])[None, :, None, None]
        bound = f8.e4m3_p_rounding_bound(q, k, v, 1.0, False, 0, 0, [0])[0, 0]
        pr = _round_e4m3_bruteforce(np.array([p2]), vals, bts)[0]
        err = abs(pr - p2) / (1.0 + p2)
        assert math.isclose(err, want_frac * bound, rel_tol=1e-9), (p2, err, bound)


def check_p_rounding_variance(f8, seed=23):
    """Brute-force rounding of P' = c P, with c = 2^u drawn per row, over many
    rows: the mean squared change of O stays below the variance bound and above
    a quarter of it (for normal values the half-unit error is between 2^-5 P
    and 2^-4 P, so the bound overstates the variance by a factor 1 to 4)."""
    bts = np.arange(127)
    vals = _torch_decode(bts)
    rng = np.random.default_rng(seed)
    Sq, Sk, D = 64, 96, 4
    q = rng.standard_normal((1, Sq, 1, D)) * 1.5
    k = rng.standard_normal((1, Sk, 1, D)) * 1.5
    v = rng.standard_normal((1, Sk, 1, D)) * 3.0
    scale = 0.8
    rows = np.arange(Sq)
    var = f8.e4m3_p_rounding_variance(q, k, v, scale, False, 0, 0, rows)
    x = scale * (q[0, :, 0] @ k[0, :, 0].T)
    p = np.exp(x - x.max(-1, keepdims=True))
    l = p.sum(-1, keepdims=True)
    o = (p @ v[0, :, 0]) / l
    c = 2.0 ** rng.uniform(0, 8, size=(Sq, 1))
    pr = _round_e4m3_bruteforce(c * p, vals, bts) / c
    err2 = (((pr @ v[0, :, 0]) / l - o) ** 2).sum()
    ratio = err2 / var.sum()
    assert 0.25 <= ratio <= 1.0, ratio


ALL_FP8_CHECKS = [
    check_e4m3_closed_forms, check_e4m3_all_bytes_vs_torch, check_e4m3_order_and_sign,
    check_attention_vs_sdpa, check_descale_algebra, check_p_rounding_bound, check_p_rounding_variance,
]
