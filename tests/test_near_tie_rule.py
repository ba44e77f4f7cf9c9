"""The acceptance rule for index sets that differ from the oracle's (host logic, no GPU)."""
import numpy as np
import pytest

from helpers import TIE_REL, near_tie_ok


def _scores(gap):
    """k = 5: candidates 0-3 clear, the k-th score tau = 1.5 at index 4, a rival at index 5
    that trails it by `gap` (relative), then small ones; max / tau = 100."""
    return np.array([150.0, 5.0, 4.0, 3.0, 1.5, 1.5 * (1 - gap), 1.0, 0.5])


def test_identical_sets_pass():
    s = _scores(0.0)
    assert near_tie_ok([0, 1, 2], [0, 1, 2], s) == 0


def test_swap_within_tau_relative_bound_passes():
    s = _scores(0.5 * TIE_REL)
    assert near_tie_ok([0, 1, 2, 3, 5], [0, 1, 2, 3, 4], s) == 2


def test_swap_beyond_tau_relative_bound_fails_even_when_small_against_the_max():
    """A gap of 3e-5 tau is 3e-7 of the largest score: the old max-relative bound let it pass."""
    s = _scores(3 * TIE_REL)
    with pytest.raises(AssertionError):
        near_tie_ok([0, 1, 2, 3, 5], [0, 1, 2, 3, 4], s)
    assert near_tie_ok([0, 1, 2, 3, 5], [0, 1, 2, 3, 4], s, relative_to="max") == 2


def test_floor_keeps_rounding_level_tau_decidable():
    """tau far below the largest score: the bound is floored at 1e-3 of it."""
    s = np.full(20, 1e-9)
    s[0] = 1.0
    s[5], s[6] = 1e-9, 1e-9 + 5e-10
    assert near_tie_ok([0, 6], [0, 5], s) == 2


def test_block_logits_straddling_zero_use_the_max_bound():
    s = np.array([3.0, -2.0, 1e-7, -1e-7, 0.5])
    assert near_tie_ok([0, 4, 3], [0, 4, 2], s, relative_to="max") == 2
    with pytest.raises(AssertionError):
        near_tie_ok([0, 4, 1], [0, 4, 2], s, relative_to="max")


def test_size_mismatch_fails():
    with pytest.raises(AssertionError):
        near_tie_ok([1, 2], [1, 2, 3], np.arange(5.0))
