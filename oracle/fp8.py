"""fp64 oracle for the e4m3 forward: decoding of E4M3 bytes and attention on
the decoded, descaled values.

TEST INFRASTRUCTURE ONLY, like ``oracle.attention``: only ``tests/``,
``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may use
it. It shares no code with the CUDA library.

The pages say only that FlashAttention-3 adds an FP8 data type on H100
([P5] sections "H100的FP8加速能力" and "未来展望：FlashAttention-3带来的新可能").
Reading used: the operation is unchanged (exact attention); Q, K and V arrive
as E4M3 bytes with one descale factor per tensor, and the result to compare
against is exact attention on the values those bytes and factors stand for.
The E4M3 format is the OCP 8-bit floating-point format: 1 sign bit, 4 exponent
bits with bias 7, 3 mantissa bits, subnormals at exponent field 0, no
infinities, and S.1111.111 as the only NaN encoding (largest finite 448).

Page legend: [P5] the FlashAttention "IO感知" overview (0539edu.com/news/165270).

Pinned by ``tests/test_oracle_pins.py`` (E4M3 decoding against the format's
closed forms and against torch's float8_e4m3fn, the descale algebra).
"""
from __future__ import annotations

import numpy as np

from .attention import attention_forward, _rows_scores, _f64


def decode_e4m3(b) -> np.ndarray:
    """E4M3 bytes (any integer array, values 0..255) -> fp64 values.

    Field by field: sign s = bit 7, exponent e = bits 6..3, mantissa m = bits
    2..0. e = 0: (-1)^s * m/8 * 2^(1-7); 0 < e: (-1)^s * (1 + m/8) * 2^(e-7),
    except e = 15 with m = 7, which is NaN.
    """
    b = np.asarray(b).astype(np.int64)
    if np.any((b < 0) | (b > 255)):
        raise ValueError("E4M3 bytes must lie in 0..255")
    s = (b >> 7) & 1
    e = (b >> 3) & 0xF
    m = b & 0x7
    mag = np.where(e == 0, (m / 8.0) * 2.0 ** (1 - 7), (1.0 + m / 8.0) * np.exp2(e - 7.0))
    mag = np.where((e == 15) & (m == 7), np.nan, mag)
    return np.where(s == 1, -mag, mag)


def dequantize(b, descale: float) -> np.ndarray:
    """Real values of an E4M3 tensor with a per-tensor descale factor."""
    return decode_e4m3(b) * float(descale)


def attention_forward_e4m3(q8, k8, v8, q_descale, k_descale, v_descale, scale: float, causal: bool):
    """O and LSE of exact attention on the dequantized inputs ([B,S,H,D] bytes)."""
    return attention_forward(dequantize(q8, q_descale), dequantize(k8, k_descale),
                             dequantize(v8, v_descale), scale, causal)


def e4m3_p_rounding_bound(q, k, v, scale: float, causal: bool, b: int, h: int, rows):
    """Worst-case change of O[b, rows, h, :] when every probability fed to the
    P V product is rounded to E4M3 while the row sum uses the unrounded values.

    With x_ij the scaled scores, P_ij = exp(x_ij - max_j x_ij) and
    l_i = sum_j P_ij, a value P' = c P (c >= 1 when P is taken relative to a
    running maximum that is at most the row maximum) rounds to the nearest
    E4M3 value with an error of at most 2^-4 P' (normal range: half a unit in
    the last of 3 mantissa bits) or 2^-10 (subnormal spacing 2^-9). Carried
    through the final division by c l, each element of O moves by at most
        sum_j max(2^-4 P_ij, 2^-10) |v_jd| / l_i.
    q, k, v are the dequantized fp64 inputs. Returns [len(rows), D].
    """
    x = _rows_scores(q, k, scale, causal, b, h, rows)            # [R, Sk], -inf where masked
    mx = np.max(x, axis=-1, keepdims=True)
    mx = np.where(np.isfinite(mx), mx, 0.0)
    p = np.exp(x - mx)
    allowed = np.isfinite(x)
    l = np.sum(p, axis=-1, keepdims=True)
    l = np.where(l > 0, l, 1.0)
    h_err = np.where(allowed, np.maximum(2.0 ** -4 * p, 2.0 ** -10), 0.0)
    return (h_err @ np.abs(_f64(v[b, :, h]))) / l



def e4m3_p_rounding_variance(q, k, v, scale: float, causal: bool, b: int, h: int, rows):
    """Upper bound on the expected squared change of O[b, rows, h, :] from the
    same rounding, modelling each rounding error as uniform on [-u, u] (variance
    u^2 / 3) and independent across keys, with u the bound on the error used by
    ``e4m3_p_rounding_bound``:
        sum_j max(2^-4 P_ij, 2^-10)^2 v_jd^2 / (3 l_i^2).
    Returns [len(rows), D].
    """
    x = _rows_scores(q, k, scale, causal, b, h, rows)
    mx = np.max(x, axis=-1, keepdims=True)
    mx = np.where(np.isfinite(mx), mx, 0.0)
    p = np.exp(x - mx)
    allowed = np.isfinite(x)
    l = np.sum(p, axis=-1, keepdims=True)
    l = np.where(l > 0, l, 1.0)
    u = np.where(allowed, np.maximum(2.0 ** -4 * p, 2.0 ** -10), 0.0)
    return ((u * u) @ (_f64(v[b, :, h]) ** 2)) / (3.0 * l * l)
