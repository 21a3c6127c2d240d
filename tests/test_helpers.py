"""The comparison helper the parity tests use (no GPU)."""
import numpy as np
import pytest

from helpers import max_abs


def test_max_abs_is_the_largest_difference():
    a = np.array([[1.0, 2.0], [3.0, 4.0]])
    b = a + np.array([[0.0, -0.25], [0.5, 0.0]])
    assert max_abs(a, b) == 0.5


def test_max_abs_skips_positions_without_a_reference():
    a = np.array([1.0, 100.0])
    b = np.array([1.0, np.nan])                    # the oracle did not compute the second unit
    assert max_abs(a, b) == 0.0


@pytest.mark.parametrize("bad", [np.nan, np.inf, -np.inf])
def test_max_abs_fails_a_non_finite_output(bad):
    a = np.array([1.0, bad])
    b = np.array([1.0, 2.0])
    assert max_abs(a, b) == float("inf")


def test_max_abs_rejects_shapes_that_differ():
    with pytest.raises(AssertionError):
        max_abs(np.zeros((2, 3)), np.zeros((3,)))
