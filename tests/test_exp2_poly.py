"""The forward kernel's software exp2 (Cody-Waite reduction + degree-3
polynomial, exp2_poly2 in csrc/sm100.cuh), emulated step by step in float32
with numpy and checked against exp2 and against the fit's error bound."""
import os
import re

import numpy as np

HDR = os.path.join(os.path.dirname(os.path.dirname(__file__)), "exact_io_aware_96_b200", "csrc", "sm100.cuh")


def coefficients():
    src = open(HDR).read()
    body = src[src.index("exp2_poly2(uint64_t t)"):]
    body = body[:body.index("\n}\n")]
    vals = [float(v) for v in re.findall(r"f2\(([0-9.]+)f, \1f\)", body)]
    c3, c2, c1, c0 = vals  # Horner order in the source: c3, c2, then c1, c0
    return np.float32(c0), np.float32(c1), np.float32(c2), np.float32(c3)


def exp2_poly(t):
    """The kernel's steps in float32 (fma rounding modelled by float64 then one float32 rounding)."""
    c0, c1, c2, c3 = coefficients()
    f32 = np.float32
    t = np.maximum(t.astype(np.float32), f32(-126.0))
    magic = f32(12582912.0)
    r = (t + magic).astype(np.float32)
    n = (r - magic).astype(np.float32)
    f = (t.astype(np.float64) - n.astype(np.float64)).astype(np.float32)  # fma(n, -1, t)
    fma = lambda a, b, c: (a.astype(np.float64) * b + c).astype(np.float32)
    p = fma(np.full_like(f, c3), f, c2)
    p = fma(p, f, c1)
    p = fma(p, f, c0)
    bits = p.view(np.uint32) + (r.view(np.uint32) << np.uint32(23))
    return bits.astype(np.uint32).view(np.float32)


def test_coefficients_parse():
    c = coefficients()
    assert abs(c[0] - 1) < 1e-3 and abs(c[1] - np.log(2)) < 1e-3


def test_relative_error_over_softmax_range():
    # arguments the softmax feeds it: s*scale*log2e - m, at most 8 (stale max), down to the clamp
    # (below -125 the result is subnormal and only its size matters; see the clamp test)
    t = np.concatenate([np.linspace(-125, 8, 2_000_001), np.linspace(-1, 1, 200_001)]).astype(np.float32)
    got = exp2_poly(t).astype(np.float64)
    ref = np.exp2(t.astype(np.float64))
    rel = np.abs(got / ref - 1)
    assert rel.max() < 8e-5, rel.max()   # fit bound 7.5e-5 plus float32 evaluation


def test_integer_arguments_exact_scale():
    t = np.arange(-125, 9, dtype=np.float32)
    got = exp2_poly(t).astype(np.float64)
    assert np.all(np.abs(got / np.exp2(t.astype(np.float64)) - 1) < 8e-5)


def test_clamp_gives_tiny_positive_not_nan():
    t = np.array([-np.inf, -1e30, -500.0, -127.0, -126.0, -125.6], dtype=np.float32)
    got = exp2_poly(t)
    assert np.all(np.isfinite(got)) and np.all(got >= 0) and np.all(got < 2.0 ** -125)
