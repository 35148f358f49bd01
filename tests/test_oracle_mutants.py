"""Plant plausible mistakes in a copy of the oracle and show the pins catch each.

Each mutant is the oracle's source with one edit (a dropped term, a wrong sign,
a wrong operand or index), loaded as a separate module on the CPU. The test
passes when at least one pin in ``oracle_checks.ALL_CHECKS`` fails on it.
"""
import os
import types

import pytest

from tests import oracle_checks as oc

SRC = os.path.join(os.path.dirname(os.path.dirname(__file__)), "oracle", "attention.py")

MUTANTS = {
    "dropped_scale": ("x = scale * (_bh(q) @ _bh(k).swapaxes(-1, -2))", "x = (_bh(q) @ _bh(k).swapaxes(-1, -2))"),
    "top_left_causal": ("return j <= i + (Sk - Sq)", "return j <= i"),
    "strict_causal": ("return j <= i + (Sk - Sq)", "return j < i + (Sk - Sq)"),
    "dx_sign": ("dx = p * (dp - dvec[..., None])", "dx = p * (dp + dvec[..., None])"),
    "dx_no_delta": ("dx = p * (dp - dvec[..., None])", "dx = p * dp"),
    "dk_wrong_operand": ("dk = scale * (dx.swapaxes(-1, -2) @ qh)", "dk = scale * (dx.swapaxes(-1, -2) @ kh)"),
    "dq_no_scale": ("dq = scale * (dx @ kh)", "dq = (dx @ kh)"),
    "dv_transposed_p": ("dv = p.swapaxes(-1, -2) @ doh", "dv = p @ doh"),
    "dp_wrong_operand": ("dp = doh @ vh.swapaxes(-1, -2)", "dp = doh @ kh.swapaxes(-1, -2)"),
    "lse_no_max": ("out = m_safe + np.log(s)", "out = np.log(s)"),
    "online_printed_update": ("o_acc = alpha[..., None] * o_acc + p @ vb", "o_acc = l[..., None] * o_acc + p @ vb"),
    "online_no_rescale_l": ("l = alpha * l + np.sum(p, axis=-1)", "l = l + np.sum(p, axis=-1)"),
    "rows_causal_offset": ("x = np.where(j <= rows[:, None] + (Sk - Sq), x, -np.inf)",
                           "x = np.where(j <= rows[:, None], x, -np.inf)"),
    "delta_wrong_tensor": ('return np.einsum("bihd,bihd->bhi", _f64(o), _f64(do))',
                           'return np.einsum("bihd,bihd->bhi", _f64(do), _f64(do))'),
}


def _load_mutant(old, new):
    src = open(SRC).read()
    assert src.count(old) == 1, old
    mod = types.ModuleType("oracle_mutant")
    exec(compile(src.replace(old, new), "oracle_mutant", "exec"), mod.__dict__)
    return mod


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name):
    mod = _load_mutant(*MUTANTS[name])
    failed = []
    for check in oc.ALL_CHECKS:
        try:
            check(mod)
        except Exception as e:  # an AssertionError or a shape error both count
            failed.append(check.__name__)
    assert failed, f"no pin caught mutant {name}"
