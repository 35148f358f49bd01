"""The e4m3 oracle (``oracle.fp8``) against its pins, and planted mistakes in a
copy of it that the pins must catch (CPU only)."""
import os
import types

import pytest

import oracle.fp8
from tests import oracle_fp8_checks as fc

SRC = os.path.join(os.path.dirname(os.path.dirname(__file__)), "oracle", "fp8.py")


@pytest.mark.parametrize("check", fc.ALL_FP8_CHECKS, ids=lambda c: c.__name__)
def test_fp8_oracle_pin(check):
    check(oracle.fp8)


MUTANTS = {
    "exponent_bias_8": ("np.exp2(e - 7.0)", "np.exp2(e - 8.0)"),
    "subnormal_scale": ("(m / 8.0) * 2.0 ** (1 - 7)", "(m / 8.0) * 2.0 ** (0 - 7)"),
    "mantissa_sixteenths": ("(1.0 + m / 8.0)", "(1.0 + m / 16.0)"),
    "no_nan": ("mag = np.where((e == 15) & (m == 7), np.nan, mag)", "mag = mag"),
    "no_sign": ("return np.where(s == 1, -mag, mag)", "return mag"),
    "descale_ignored": ("return decode_e4m3(b) * float(descale)", "return decode_e4m3(b)"),
    "v_takes_k_descale": ("dequantize(v8, v_descale), scale, causal)", "dequantize(v8, k_descale), scale, causal)"),
    "bound_half_ulp_2m5": ("h_err = np.where(allowed, np.maximum(2.0 ** -4 * p, 2.0 ** -10), 0.0)",
                           "h_err = np.where(allowed, np.maximum(2.0 ** -5 * p, 2.0 ** -10), 0.0)"),
    "bound_no_subnormal": ("h_err = np.where(allowed, np.maximum(2.0 ** -4 * p, 2.0 ** -10), 0.0)",
                           "h_err = np.where(allowed, 2.0 ** -4 * p, 0.0)"),
    "variance_half_ulp_2m5": ("u = np.where(allowed, np.maximum(2.0 ** -4 * p, 2.0 ** -10), 0.0)",
                              "u = np.where(allowed, np.maximum(2.0 ** -5 * p, 2.0 ** -10), 0.0)"),
    "bound_signed_v": ("(h_err @ np.abs(_f64(v[b, :, h]))) / l", "(h_err @ _f64(v[b, :, h])) / l"),
    "variance_no_third": ("/ (3.0 * l * l)", "/ (l * l)"),
    "variance_not_squared": ("((u * u) @ (_f64(v[b, :, h]) ** 2))", "((u * u) @ np.abs(_f64(v[b, :, h])))"),
    "variance_one_l": ("/ (3.0 * l * l)", "/ (3.0 * l)"),
    "bound_no_l": ("(h_err @ np.abs(_f64(v[b, :, h]))) / l", "(h_err @ np.abs(_f64(v[b, :, h])))"),
}


def _load_mutant(old, new):
    src = open(SRC).read()
    assert src.count(old) == 1, old
    src = src.replace(old, new).replace("from .attention import", "from oracle.attention import")
    mod = types.ModuleType("oracle_fp8_mutant")
    exec(compile(src, "oracle_fp8_mutant", "exec"), mod.__dict__)
    return mod


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_fp8_mutant_is_caught(name):
    mod = _load_mutant(*MUTANTS[name])
    failed = []
    for check in fc.ALL_FP8_CHECKS:
        try:
            check(mod)
        except Exception:
            failed.append(check.__name__)
    assert failed, f"no pin caught mutant {name}"
