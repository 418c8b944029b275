"""Lloyd-Max scalar codebooks for the known post-rotation coordinate law.

Oracle module (test infrastructure only).

Pages: wis-web.com llama.cpp-fork post (PolarQuant paragraph: after the
rotation the coordinate distribution is known in advance, so it compresses
without stored quantisation constants; turbo2/3/4 modes = 2, 3, 4 bits) and the
leviatan.io article, "Benchmarks de memoire" (no additional per-value overhead).

Readings taken where the pages are silent:

* The "known law" is the exact marginal of one coordinate of a uniformly random
  unit vector in R^d: f(t) proportional to (1 - t^2)^((d-3)/2) on [-1, 1], i.e.
  t = 2B - 1 with B ~ Beta((d-1)/2, (d-1)/2). The rotated, norm-divided vector is
  exactly such a point when the input is isotropic; N(0, 1/d) is its d -> inf
  limit (kept as a separate density for the textbook pin).
* The codebook is the scalar Lloyd-Max quantiser of that law with 2**b levels,
  symmetric about 0, found by Lloyd's fixed-point iteration in double precision
  started at the level quantiles.
* Stored centroids are the Lloyd-Max values rounded to fp16 (nearest even);
  decision thresholds are the exact midpoints of adjacent stored centroids
  (exactly representable in fp32). A value equal to a threshold goes to the
  lower cell.
"""

from dataclasses import dataclass

import numpy as np
from scipy import special


class SphereMarginal:
    """Law of one coordinate of a uniform point on the unit sphere S^(d-1)."""

    def __init__(self, d: int):
        self.d = d
        self.alpha = (d - 1) / 2.0          # Beta parameters of (t + 1) / 2
        self.k = (d - 3) / 2.0              # exponent of (1 - t^2)
        self.norm = special.beta(0.5, self.k + 1.0)  # integral of (1-t^2)^k over [-1,1]
        self.upper = 1.0

    def tail(self, x):
        """P(t > x)."""
        x = np.asarray(x, dtype=np.float64)
        return special.betaincc(self.alpha, self.alpha, np.clip((x + 1.0) / 2.0, 0.0, 1.0))

    def moment1(self, a, b):
        """Integral of t f(t) over (a, b): closed form of (1-t^2)^(k+1) / (-2(k+1))."""
        a = np.asarray(a, dtype=np.float64)
        b = np.asarray(b, dtype=np.float64)
        k1 = self.k + 1.0
        fa = np.power(np.clip(1.0 - a * a, 0.0, None), k1)
        fb = np.power(np.clip(1.0 - b * b, 0.0, None), k1)
        return (fa - fb) / (2.0 * k1 * self.norm)

    def moment2(self, a, b):
        """Integral of t^2 f(t) over (a, b), using t^2 (1-t^2)^k = (1-t^2)^k - (1-t^2)^(k+1)."""
        nxt = SphereMarginal(self.d + 2)   # exponent k + 1, Beta parameter alpha + 1
        mass_k = self.tail(a) - self.tail(b)
        mass_k1 = nxt.tail(a) - nxt.tail(b)
        return mass_k - mass_k1 * nxt.norm / self.norm

    def quantile(self, p):
        return 2.0 * special.betaincinv(self.alpha, self.alpha, p) - 1.0

    def second_moment(self):
        return 1.0 / self.d


class StandardNormal:
    """N(0, 1): used only to pin the Lloyd iteration against Max's (1960) table."""

    upper = np.inf

    def tail(self, x):
        return special.ndtr(-np.asarray(x, dtype=np.float64))

    def moment1(self, a, b):
        phi = lambda t: np.exp(-0.5 * np.square(t)) / np.sqrt(2.0 * np.pi)  # noqa: E731
        return phi(np.asarray(a, dtype=np.float64)) - phi(np.asarray(b, dtype=np.float64))

    def moment2(self, a, b):
        a = np.asarray(a, dtype=np.float64)
        b = np.asarray(b, dtype=np.float64)
        phi = lambda t: np.where(np.isinf(t), 0.0, np.exp(-0.5 * np.square(t)) / np.sqrt(2.0 * np.pi))  # noqa: E731
        ta = np.where(np.isinf(a), 0.0, a)
        tb = np.where(np.isinf(b), 0.0, b)
        return (ta * phi(a) - tb * phi(b)) + (self.tail(a) - self.tail(b))

    def quantile(self, p):
        return special.ndtri(p)

    def second_moment(self):
        return 1.0


def lloyd_max_positive(density, levels: int, max_iter: int = 200000):
    """Positive-half Lloyd-Max centroids of a symmetric density with 2*levels cells.

    Cells of the positive half are (0, b1), (b1, b2), ..., (b_{L-1}, upper) with
    b_j the midpoint of adjacent centroids; each centroid is the conditional mean
    of its cell. Iterates until the largest change is a few ulps of the largest centroid and
    stops shrinking.
    Returns (centroids, iterations).
    """
    p = 0.5 + (np.arange(levels) + 0.5) / (2.0 * levels)
    c = np.asarray(density.quantile(p), dtype=np.float64)
    it = 0
    stall = 0
    best = np.inf
    for it in range(1, max_iter + 1):
        bnd = np.concatenate(([0.0], 0.5 * (c[:-1] + c[1:]), [density.upper]))
        mass = density.tail(bnd[:-1]) - density.tail(bnd[1:])
        c_new = density.moment1(bnd[:-1], bnd[1:]) / mass
        delta = float(np.max(np.abs(c_new - c)))
        c = c_new
        # converged once the step is a few ulps of the largest centroid and stops shrinking
        if delta <= 16.0 * np.finfo(np.float64).eps * float(np.max(np.abs(c))):
            stall = stall + 1 if delta >= best else 0
            best = min(best, delta)
            if delta == 0.0 or stall >= 3:
                break
    return c, it


@dataclass
class Codebook:
    bits: int
    centroids: np.ndarray        # ascending, fp16 values held in float64
    thresholds: np.ndarray       # 2**bits - 1 midpoints, fp32-exact, float64
    centroids_exact: np.ndarray  # the un-rounded Lloyd-Max values (float64)


def codebook(bits: int, d: int = 128, density=None) -> Codebook:
    """Stored b-bit codebook for head dimension d (sphere marginal unless told otherwise)."""
    if density is None:
        density = SphereMarginal(d)
    pos, _ = lloyd_max_positive(density, 2 ** (bits - 1))
    exact = np.concatenate((-pos[::-1], pos))
    c16 = exact.astype(np.float16).astype(np.float64)
    thr = 0.5 * (c16[:-1] + c16[1:])
    if not np.array_equal(thr.astype(np.float32).astype(np.float64), thr):
        raise AssertionError("threshold not representable in fp32")
    return Codebook(bits, c16, thr, exact)


def encode(y: np.ndarray, thresholds: np.ndarray) -> np.ndarray:
    """Code of each value: the number of thresholds strictly below it (ties go down)."""
    y = np.asarray(y, dtype=np.float64)
    return np.sum(y[..., None] > thresholds, axis=-1).astype(np.int64)


def distortion(density, centroids: np.ndarray) -> float:
    """E[(t - Q(t))^2] for nearest-centroid quantisation with the given (ascending) centroids."""
    c = np.asarray(centroids, dtype=np.float64)
    lo = -density.upper
    bnd = np.concatenate(([lo], 0.5 * (c[:-1] + c[1:]), [density.upper]))
    a, b = bnd[:-1], bnd[1:]
    m0 = density.tail(a) - density.tail(b)
    m1 = density.moment1(a, b)
    m2 = density.moment2(a, b)
    return float(np.sum(m2 - 2.0 * c * m1 + c * c * m0))
