"""Natural-order (Sylvester) Walsh-Hadamard transform and the random rotation.

Oracle module (test infrastructure only).

wis-web.com llama.cpp-fork post, PolarQuant paragraph: a Walsh-Hadamard
rotation is applied to each vector so that its coordinates follow a known law.
The rotation used is R = H D / sqrt(d), with H the +-1 Sylvester Hadamard matrix
and D a seeded random sign diagonal; R is orthogonal and R^T = D H / sqrt(d).
"""

import numpy as np


def fwht(x: np.ndarray) -> np.ndarray:
    """Unnormalised Walsh-Hadamard transform H x along the last axis (natural order).

    Butterflies of width 1, 2, 4, ...: (a, b) -> (a + b, a - b). The length must
    be a power of two.
    """
    x = np.array(x, dtype=np.float64, copy=True)
    n = x.shape[-1]
    if n & (n - 1):
        raise ValueError("length must be a power of two")
    lead = x.shape[:-1]
    h = 1
    while h < n:
        v = x.reshape(lead + (n // (2 * h), 2, h))
        a = v[..., 0, :].copy()
        b = v[..., 1, :].copy()
        v[..., 0, :] = a + b
        v[..., 1, :] = a - b
        h *= 2
    return x


def rotate(x: np.ndarray, signs: np.ndarray) -> np.ndarray:
    """R x = H (D x) / sqrt(d) along the last axis."""
    d = x.shape[-1]
    return fwht(np.asarray(x, dtype=np.float64) * signs) / np.sqrt(d)


def unrotate(y: np.ndarray, signs: np.ndarray) -> np.ndarray:
    """R^T y = D (H y) / sqrt(d) along the last axis."""
    d = y.shape[-1]
    return signs * fwht(y) / np.sqrt(d)
