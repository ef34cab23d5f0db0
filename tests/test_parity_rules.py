"""The top-k comparison rule of the GPU parity tests, checked on hand-made rows
(CPU): it accepts a different choice inside the tie band and rejects every
other kind of difference."""
import numpy as np
import pytest

from parity import check_topk


def _row(scores):
    return np.asarray(scores, dtype=np.float64)[None, :]


def test_identical_sets_pass():
    s = _row([1.0, 5.0, 3.0, -np.inf])
    same = check_topk(np.array([[1, 2]]), s, np.array([[1, 2]]), 2, "t")
    assert same.all()


def test_swap_inside_the_tie_band_passes():
    # s_2 = 5 and s_3 = 5 - 1e-6 tie within 1e-3 relative: {0, 1} and {0, 2} are both top-2 sets
    s = _row([10.0, 5.0, 5.0 - 1e-6, 1.0])
    same = check_topk(np.array([[0, 2]]), s, np.array([[0, 1]]), 2, "t")
    assert not same.any()


def test_dropping_an_entry_above_the_band_fails():
    # scores 10, 5, 5 - eps: the set {1, 2} leaves out the clear winner 0
    s = _row([10.0, 5.0, 5.0 - 1e-6, 1.0])
    with pytest.raises(AssertionError, match="above the band"):
        check_topk(np.array([[1, 2]]), s, np.array([[0, 1]]), 2, "t")


def test_difference_outside_the_band_fails():
    s = _row([10.0, 5.0, 4.0, 1.0])
    with pytest.raises(AssertionError, match="outside the tie band"):
        check_topk(np.array([[0, 2]]), s, np.array([[0, 1]]), 2, "t")


def test_invisible_or_unordered_or_padded_selections_fail():
    s = _row([10.0, 5.0, 5.0 - 1e-6, -np.inf, 5.0 - 2e-6])
    with pytest.raises(AssertionError, match="invisible"):
        check_topk(np.array([[0, 3]]), s, np.array([[0, 1]]), 2, "t")
    with pytest.raises(AssertionError, match="ascending"):
        check_topk(np.array([[2, 0]]), s, np.array([[0, 1]]), 2, "t")
    with pytest.raises(AssertionError, match="padding"):
        check_topk(np.array([[0, -1]]), s, np.array([[0, 1]]), 2, "t")


def test_rows_with_every_visible_entry_must_match_exactly():
    s = _row([1.0, 2.0, -np.inf, -np.inf])
    with pytest.raises(AssertionError, match="every visible entry fits"):
        check_topk(np.array([[0, -1, -1]]), s, np.array([[0, 1, -1]]), 3, "t")
