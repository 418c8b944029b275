"""Pins of the natural-order Walsh-Hadamard transform and the rotation."""
import numpy as np
import pytest
from scipy.linalg import hadamard

from oracle.hadamard import fwht, rotate, unrotate
from oracle.rng import sign_vector


@pytest.mark.parametrize("n", [2, 4, 8, 16, 128])
def test_fwht_equals_sylvester_matrix(n):
    x = np.random.default_rng(n).standard_normal((3, n))
    np.testing.assert_allclose(fwht(x), x @ hadamard(n).T, rtol=0, atol=1e-12)


@pytest.mark.parametrize("n", [2, 4, 8, 16])
def test_hadamard_orthogonality_exact(n):
    h = fwht(np.eye(n))
    assert np.array_equal(h @ h.T, n * np.eye(n))


def test_fwht_round_trip_exact_on_integers():
    x = np.random.default_rng(0).integers(-1000, 1000, size=(5, 128)).astype(np.float64)
    assert np.array_equal(fwht(fwht(x)), 128 * x)


def test_rotation_is_orthogonal():
    d = sign_vector(3, 128)
    x = np.random.default_rng(1).standard_normal((10, 128))
    y = rotate(x, d)
    np.testing.assert_allclose(np.linalg.norm(y, axis=1), np.linalg.norm(x, axis=1), rtol=1e-15)
    np.testing.assert_allclose(unrotate(y, d), x, rtol=0, atol=1e-14)
    r = rotate(np.eye(128), d)          # rows R e_i -> R^T as a matrix
    np.testing.assert_allclose(r @ r.T, np.eye(128), atol=1e-14)


def test_fwht_rejects_non_power_of_two():
    with pytest.raises(ValueError):
        fwht(np.ones(12))
