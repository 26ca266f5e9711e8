"""The parity checkers themselves, on CPU: a valid answer passes and each kind
of wrong answer fails (so a GPU result cannot slip through a lax check)."""
import numpy as np
import pytest

from helpers import check_topk_valid


def _scores():
    # ids 0..9; scores with an exact tie at the k = 4 boundary (ids 3 and 7)
    return np.array([9.0, 8.0, 7.0, 5.0, 1.0, 0.5, 0.25, 5.0, -1.0, 6.0])


def test_topk_valid_accepts_either_side_of_a_tie():
    s = _scores()
    check_topk_valid(np.array([0, 1, 2, 9]), s, 4)          # no tie involved (k = 4: 9, 8, 7, 6)
    check_topk_valid(np.array([0, 1, 2, 3, 9]), s, 5)       # tie 3 / 7 at k = 5: lower index
    check_topk_valid(np.array([0, 1, 2, 7, 9]), s, 5)       # the other side of the same tie


@pytest.mark.parametrize("ids,k,why", [
    ([0, 1, 2, 4, 9], 5, "kept a low id"),
    ([0, 1, 3, 7, 9], 5, "dropped an id above the boundary"),
    ([0, 2, 1, 3, 9], 5, "not ascending"),
    ([0, 1, 2, 3], 5, "too few ids"),
    ([0, 1, 2, 3, 3], 5, "duplicate id"),
    ([0, 1, 2, 3, 10], 5, "out of range"),
])
def test_topk_valid_rejects_wrong_answers(ids, k, why):
    with pytest.raises(AssertionError):
        check_topk_valid(np.array(ids), _scores(), k, why)
