"""The bench line's sampled decode check on CPU: errors against the oracle's outputs,
and non-finite outputs counted as failures (a NaN compares as no error in a maximum)."""
import os
import sys

import numpy as np

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402


def _want(heads=4, seed=0):
    return np.random.default_rng(seed).standard_normal((heads, 128))


def test_identical_outputs_have_no_error():
    want = _want()
    assert bench.decode_row_errors(want.copy(), want) == (0.0, 0.0, 0)


def test_one_wrong_element_shows_in_the_element_error():
    want = _want()
    got = want.copy()
    got[2, 17] += 0.01 * np.linalg.norm(want[2])
    worst, worst_e, nonfinite = bench.decode_row_errors(got, want)
    assert nonfinite == 0
    assert abs(worst - 0.01) < 1e-12          # per head: the error's norm over the head's
    floor = np.linalg.norm(want[2]) / np.sqrt(128)
    assert abs(worst_e - 0.01 * np.linalg.norm(want[2]) / max(abs(want[2, 17]), floor)) < 1e-9


def test_non_finite_outputs_are_counted():
    want = _want()
    got = want.copy()
    got[0, 3] = np.nan
    got[1, 5] = np.inf
    worst, worst_e, nonfinite = bench.decode_row_errors(got, want)
    assert nonfinite == 2
    # a NaN must not read as a perfect match
    assert not (nonfinite == 0 and worst <= 1e-3)
