"""The per-block gradient check (tests/parity.py) catches an error that the
whole-tensor relative L2 misses.

The fault is planted on the CPU in the oracle's own result, not in a kernel:
the dK rows of one 128-key block lose the contribution of one 128-row query
block, which is what a kernel that skipped one (query block, key block) pair
would return. It is built from two oracle calls: the full dK, and dK with
dO = 0 on that query block (whose rows then contribute nothing), spliced in
on that key block only. On one head of 4096 rows the whole-tensor error stays
under the 5e-2 bar while that block's error is several times over it.
"""
import numpy as np
import pytest

import oracle
from tests.parity import GRAD_TOL, blocks_rel_l2, check_grad, rel_l2

S, D, QB, KB = 4096, 64, 11, 20


def _planted():
    rng = np.random.default_rng(7)
    q, k, v, do = (rng.standard_normal((1, S, 1, D)).astype(np.float16).astype(np.float64) for _ in range(4))
    scale = D ** -0.5
    _, dk, _, _ = oracle.attention_backward(q, k, v, do, scale, False)
    do0 = do.copy()
    do0[:, QB * 128:(QB + 1) * 128] = 0.0
    _, dk0, _, _ = oracle.attention_backward(q, k, v, do0, scale, False)
    bad = dk.copy()
    bad[:, KB * 128:(KB + 1) * 128] = dk0[:, KB * 128:(KB + 1) * 128]
    return dk, bad


def test_block_check_catches_one_missing_block_pair():
    dk, bad = _planted()
    whole = rel_l2(bad, dk)
    assert whole < GRAD_TOL / 1.5, f"the planted fault should pass the whole-tensor bar, got {whole:.3e}"
    check_grad(bad, dk, "whole tensor only")  # passes: the fault hides in the norm of the rest
    errs = dict(blocks_rel_l2(bad, dk, row_axis=1, head_axes=(0, 2)))
    worst = max(errs, key=errs.get)
    assert worst == ((0, 0), KB * 128) and errs[worst] > 2 * GRAD_TOL
    assert all(e == 0.0 for key, e in errs.items() if key != worst)
    with pytest.raises(AssertionError, match="rows from 2560"):
        check_grad(bad, dk, "per block", row_axis=1, head_axes=(0, 2))
    check_grad(dk, dk, "unperturbed", row_axis=1, head_axes=(0, 2))


def test_sampled_rows_are_checked_per_head():
    rng = np.random.default_rng(5)
    ref = rng.standard_normal((3, 40, 8))
    got = ref.copy()
    # one sampled row off by 7% of its head's norm: 4% of the whole tensor
    got[1, 7] += 0.07 * np.linalg.norm(ref[1]) / np.sqrt(ref.shape[2])
    check_grad(got, ref, "whole tensor only")
    with pytest.raises(AssertionError, match="head index \\(1,\\)"):
        check_grad(got, ref, "sampled", row_axis=1, head_axes=(0,), rows="sampled")
    got = ref.copy()
    got[1, 7] += 0.03 * np.linalg.norm(ref[1]) / np.sqrt(ref.shape[2])
    check_grad(got, ref, "sampled", row_axis=1, head_axes=(0,), rows="sampled")


def test_block_check_groups_sampled_rows_and_floors_near_zero_pieces():
    rng = np.random.default_rng(3)
    ref = rng.standard_normal((2, 40, 8))
    rows = np.sort(rng.choice(1000, size=40, replace=False))
    got = ref.copy()
    # a piece whose reference is almost zero is judged against a small share
    # of the whole norm rather than its own
    ref[1, rows // 128 == rows[0] // 128] *= 1e-9
    got[1, rows // 128 == rows[0] // 128] = 1e-6
    check_grad(got, ref, "near-zero piece", row_axis=1, head_axes=(0,), rows=rows)
    # an error of 10% of its block's norm on one sampled row: 2.5% of the whole
    nb = np.linalg.norm(ref[0, rows // 128 == rows[5] // 128])
    got[0, 5] += 0.1 * nb / np.sqrt(ref.shape[2])
    with pytest.raises(AssertionError, match=f"head index \\(0,\\), rows from {rows[5] // 128 * 128}"):
        check_grad(got, ref, "one bad sampled row", row_axis=1, head_axes=(0,), rows=rows)
