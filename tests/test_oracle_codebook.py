"""Pins of the Lloyd-Max codebooks: textbook table, closed forms, fixed point, brute force."""
import json
import os

import numpy as np
import pytest
from scipy import integrate, special

from oracle import codebook as cb

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_gaussian_special_case_reproduces_max_1960(bits):
    ref = json.load(open(os.path.join(GOLDEN, "max1960_gaussian_levels.json")))
    pos, _ = cb.lloyd_max_positive(cb.StandardNormal(), 2 ** (bits - 1))
    want = np.array(ref["levels"][str(bits)])
    unit = 10.0 ** (np.floor(np.log10(np.abs(want))) - 3)     # last printed digit
    assert np.all(np.abs(pos - want) <= unit)


def test_one_bit_closed_forms():
    d = 128
    pos, _ = cb.lloyd_max_positive(cb.SphereMarginal(d), 1)
    e_abs = special.gamma(d / 2) / (np.sqrt(np.pi) * special.gamma((d + 1) / 2))
    assert abs(pos[0] - e_abs) < 1e-14
    g, _ = cb.lloyd_max_positive(cb.StandardNormal(), 1)
    assert abs(g[0] - np.sqrt(2 / np.pi)) < 1e-14
    # distortion of the 1-bit Gaussian quantiser is 1 - 2/pi
    assert abs(cb.distortion(cb.StandardNormal(), np.array([-g[0], g[0]])) - (1 - 2 / np.pi)) < 1e-13


def test_sphere_marginal_density_normalised_and_second_moment():
    sm = cb.SphereMarginal(128)
    f = lambda t: (1 - t * t) ** sm.k / sm.norm  # noqa: E731
    tot, _ = integrate.quad(f, -1, 1, epsabs=1e-13, epsrel=1e-13, points=[0])
    assert abs(tot - 1) < 1e-12
    m2, _ = integrate.quad(lambda t: t * t * f(t), -1, 1, epsabs=1e-15, epsrel=1e-13, points=[0])
    assert abs(m2 - 1 / 128) < 1e-13
    assert abs(sm.tail(0.0) - 0.5) < 1e-15


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_fixed_point_by_independent_quadrature(bits):
    """Each centroid is the conditional mean of its cell (adaptive quadrature, not betainc)."""
    sm = cb.SphereMarginal(128)
    pos, _ = cb.lloyd_max_positive(sm, 2 ** (bits - 1))
    f = lambda t: (1 - t * t) ** sm.k  # noqa: E731
    bnd = np.concatenate(([0.0], 0.5 * (pos[:-1] + pos[1:]), [1.0]))
    for j in range(len(pos)):
        a, b = bnd[j], bnd[j + 1]
        m0, _ = integrate.quad(f, a, b, epsabs=0, epsrel=1e-13, limit=200)
        m1, _ = integrate.quad(lambda t: t * f(t), a, b, epsabs=0, epsrel=1e-13, limit=200)
        assert abs(m1 / m0 - pos[j]) < 1e-12 * max(1.0, pos[j])


@pytest.mark.parametrize("bits", [2, 3])
def test_brute_force_sample_lloyd_agrees(bits):
    d = 128
    sm = cb.SphereMarginal(d)
    pos, _ = cb.lloyd_max_positive(sm, 2 ** (bits - 1))
    rng = np.random.default_rng(bits)
    t = np.abs(2 * rng.beta(sm.alpha, sm.alpha, size=2_000_000) - 1)   # positive half by symmetry
    c = sm.quantile(0.5 + (np.arange(len(pos)) + 0.5) / (2 * len(pos)))
    for _ in range(400):
        bnd = 0.5 * (c[:-1] + c[1:])
        idx = np.searchsorted(bnd, t)
        c = np.bincount(idx, weights=t, minlength=len(c)) / np.bincount(idx, minlength=len(c))
    # Monte-Carlo error of a conditional mean ~ std(cell)/sqrt(count); allow 6 sigma
    idx = np.searchsorted(0.5 * (pos[:-1] + pos[1:]), t)
    for j in range(len(pos)):
        cell = t[idx == j]
        assert abs(c[j] - pos[j]) < 6 * cell.std() / np.sqrt(cell.size) + 1e-6


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_perturbing_any_centroid_raises_distortion(bits):
    sm = cb.SphereMarginal(128)
    book = cb.codebook(bits)
    base = cb.distortion(sm, book.centroids_exact)
    for j in range(2 ** bits):
        for eps in (-1e-4, 1e-4):
            c = book.centroids_exact.copy()
            c[j] += eps
            assert cb.distortion(sm, np.sort(c)) > base


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_stored_tables(bits):
    book = cb.codebook(bits)
    c = book.centroids
    assert np.array_equal(c.astype(np.float16).astype(np.float64), c)
    assert np.all(np.diff(c) > 0)
    assert np.array_equal(c, -c[::-1])
    assert np.array_equal(book.thresholds, 0.5 * (c[:-1] + c[1:]))
    assert np.array_equal(book.thresholds.astype(np.float32).astype(np.float64), book.thresholds)
    assert book.thresholds[len(book.thresholds) // 2] == 0.0
    # rounding to fp16 moves each centroid by at most half an fp16 ulp
    ulp = np.spacing(np.abs(book.centroids_exact).astype(np.float16)).astype(np.float64)
    assert np.all(np.abs(c - book.centroids_exact) <= 0.5 * ulp)


def test_encode_tie_rule_and_extremes():
    book = cb.codebook(3)
    thr = book.thresholds
    assert list(cb.encode(thr, thr)) == list(range(7))            # equal -> lower cell
    assert list(cb.encode(np.nextafter(thr, 1), thr)) == list(range(1, 8))
    assert cb.encode(np.array([-1.0, 1.0]), thr).tolist() == [0, 7]


def test_encode_is_nearest_centroid():
    book = cb.codebook(4)
    y = np.random.default_rng(5).standard_normal(20000) / np.sqrt(128)
    code = cb.encode(y, book.thresholds)
    brute = np.argmin(np.abs(y[:, None] - book.centroids[None]), axis=1)
    assert np.array_equal(code, brute)


@pytest.mark.parametrize("bits", [2, 3])
def test_mse_on_uniform_sphere_points_matches_distortion(bits):
    """For isotropic x, y = R x / |x| is uniform on the sphere: E|y - c|^2 = d * D(c)."""
    from oracle.quantize import quantize
    from oracle.rng import sign_vector
    d = 128
    book = cb.codebook(bits)
    x = np.random.default_rng(bits + 10).standard_normal((20000, d))
    qz = quantize(x, sign_vector(9, d), book.centroids, book.thresholds)
    err = np.sum((qz.y - book.centroids[qz.codes]) ** 2, axis=1)
    want = d * cb.distortion(cb.SphereMarginal(d), book.centroids)
    assert abs(err.mean() - want) < 6 * err.std() / np.sqrt(err.size)
