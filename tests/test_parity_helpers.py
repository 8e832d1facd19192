"""Host-side checks of the parity comparison itself (tests/parity.py): a GPU
row must be a strictly ascending list of distinct in-range tiles, a swap is
tolerated only inside the tie band, and the tie band is reported."""
import numpy as np
import pytest

from parity import TieBandReport, assert_selection, compare_selection


def _planted(s):
    """One (b, h, query tile) row with scores s_j exactly: qhat = e0, khat_j = s_j e0."""
    s = np.asarray(s, float)
    qhat = np.zeros((1, 1, 1, 2))
    qhat[0, 0, 0, 0] = 1.0
    khat = np.zeros((1, 1, len(s), 2))
    khat[0, 0, :, 0] = s
    return qhat, khat


def _compare(oracle_mod, s, k, gpu_row):
    qhat, khat = _planted(s)
    idx, kth, _ = oracle_mod.select(qhat, khat, k)
    gpu = np.asarray(gpu_row, np.int32).reshape(1, 1, 1, k)
    return idx, compare_selection(oracle_mod, gpu, idx, kth, qhat, khat)


def test_identical_rows_pass(oracle_mod):
    idx, rep = _compare(oracle_mod, [5, 1, 9, 3], 2, [0, 2])
    assert idx.reshape(-1).tolist() == [0, 2]
    assert rep.mismatched == 0 and not rep.violations and not rep.tie_band


def test_same_set_in_another_order_is_a_violation(oracle_mod):
    _, rep = _compare(oracle_mod, [5, 1, 9, 3], 2, [2, 0])
    assert rep.violations == [0]
    with pytest.raises(AssertionError):
        assert_selection(rep, "reordered")


def test_duplicate_or_out_of_range_tiles_are_violations(oracle_mod):
    assert _compare(oracle_mod, [5, 1, 9, 3], 2, [2, 2])[1].violations == [0]
    assert _compare(oracle_mod, [5, 1, 9, 3], 2, [2, 4])[1].violations == [0]
    assert _compare(oracle_mod, [5, 1, 9, 3], 2, [-1, 2])[1].violations == [0]


def test_swap_outside_the_band_is_a_violation(oracle_mod):
    _, rep = _compare(oracle_mod, [5, 1, 9, 3], 2, [2, 3])     # 3 scores 3, the k-th scores 5
    assert rep.violations == [0] and not rep.tie_band


def test_swap_inside_the_band_is_reported(oracle_mod):
    s = [5.0, 1.0, 9.0, 5.0 * (1 - 5e-5)]                       # tiles 0 and 3 within 1e-4 relative
    _, rep = _compare(oracle_mod, s, 2, [2, 3])
    assert rep.tie_band == [0] and not rep.violations
    with pytest.warns(TieBandReport):
        assert_selection(rep, "near tie")
