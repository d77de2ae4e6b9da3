"""The parity helpers' exact-tie test, pinned on hand-built rows (CPU).

A flip between the GPU and the oracle is exempt from the flip-rate budget
only at an exact tie: (y - m) / s a half-integer in real arithmetic.  These
rows are built in the rotated domain from small integers, so which codes sit
at exact ties is known by construction."""
import numpy as np

from oracle import kvarn_oracle as O
from _parity import exact_half_ties


def _row_from_rotated(y: np.ndarray, block=None) -> np.ndarray:
    # x = y H / b: then x H / sqrt(b) = y / sqrt(b), whose (y - m) / s is that of y
    d = y.shape[-1]
    h = O.block_hadamard_matrix(d, block or d).astype(np.float64)
    return (y @ h) / (block or d)


def test_exact_ties_found_where_built():
    d = 128
    y = np.ones(d)
    y[0], y[1] = 0.0, 2.0                      # m = 0, max = 2
    x = _row_from_rotated(y).reshape(1, 1, d)
    # 2 bits: (y - m) / s = 3 y / 2 -> 1.5 at every y = 1 (a tie), 0 and 3 at the ends
    idx = (np.zeros(4, int), np.zeros(4, int), np.array([0, 1, 2, 77]))
    assert list(exact_half_ties(x, 2, 0, None, idx)) == [False, False, True, True]
    # 4 bits: 15 y / 2 -> 7.5 at y = 1: still a tie; 3 bits: 7 y / 2 -> 3.5: a tie
    assert exact_half_ties(x, 4, 0, None, idx)[2] and exact_half_ties(x, 3, 0, None, idx)[3]
    # with normalisation rounds no tie is exact
    assert not exact_half_ties(x, 2, 4, None, idx).any()


def test_near_ties_are_not_exact():
    d = 128
    y = np.ones(d)
    y[0], y[1] = 0.0, 3.0                      # 2 bits: (y - m) / s = y -> integers, no tie
    x = _row_from_rotated(y).reshape(1, 1, d)
    assert not exact_half_ties(x, 2, 0, None, (np.array([0]), np.array([0]), np.array([5]))).any()
    y = np.ones(d)
    y[0], y[1], y[2] = 0.0, 2.0, 1.0 + 2.0 ** -20   # one ulp-sized step off the tie
    x = _row_from_rotated(y).reshape(1, 1, d)
    assert list(exact_half_ties(x, 2, 0, None, (np.zeros(2, int), np.zeros(2, int), np.array([2, 3])))) == \
        [False, True]


def test_exact_ties_under_a_block_diagonal_rotation():
    d, b = 128, 32
    y = np.full(d, 4.0)
    y[0], y[40] = 0.0, 8.0                     # m = 0, max = 8: 4 bits -> 15 * 4 / 8 = 7.5
    x = _row_from_rotated(y, b).reshape(1, 1, d)
    assert exact_half_ties(x, 4, 0, b, (np.array([0]), np.array([0]), np.array([100])))[0]
    assert not exact_half_ties(x, 4, 0, b, (np.array([0]), np.array([0]), np.array([40])))[0]
