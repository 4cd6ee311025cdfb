"""Pins of the PolarQuant oracle ("TurboQuant и PolarQuant", sections "Полярное преобразование",
"Шаг 3: построение кодовых книг", "Степень сжатия").

Each check fixes a result by something other than the oracle's own formulas: block norms
computed directly, the page's worked bit count, the closed-form Lloyd solution of a uniform
density, the page's normalising constant against an independent adaptive quadrature, Monte
Carlo angles of Gaussian sub-vectors, and the page's statement that centroids lean towards
pi/4."""

import os

import numpy as np
import pytest
from scipy import integrate

from oracle import params, polar

D = 128
GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_radii_are_block_norms_and_angles_their_ratios():
    y = np.random.default_rng(0).standard_normal((50, D))
    angles, radii = polar.polar_transform(y, 4)
    for level in range(1, 5):
        blocks = y.reshape(50, D >> level, 1 << level)
        norms = np.linalg.norm(blocks, axis=2)  # radius of level l: norm of 2^l consecutive coordinates
        half = 1 << (level - 1)
        lo = np.linalg.norm(blocks[:, :, :half], axis=2)
        hi = np.linalg.norm(blocks[:, :, half:], axis=2)
        if level == 4:
            np.testing.assert_allclose(radii, norms, rtol=1e-13)
        if level >= 2:
            np.testing.assert_allclose(np.tan(angles[level - 1]), hi / lo, rtol=1e-11)
            assert angles[level - 1].min() >= 0 and angles[level - 1].max() <= np.pi / 2
    # level 1: the angle of the pair (y_2i, y_2i+1) in [0, 2 pi)
    th = angles[0]
    assert th.min() >= 0 and th.max() < 2 * np.pi
    np.testing.assert_allclose(np.cos(th) * np.hypot(y[:, 0::2], y[:, 1::2]), y[:, 0::2], atol=1e-12)
    np.testing.assert_allclose(np.sin(th) * np.hypot(y[:, 0::2], y[:, 1::2]), y[:, 1::2], atol=1e-12)
    # the transform keeps the norm in its last radii, and the inverse restores the coordinates
    np.testing.assert_allclose(np.linalg.norm(radii, axis=1), np.linalg.norm(y, axis=1), rtol=1e-13)
    np.testing.assert_allclose(polar.inverse_polar(angles, radii), y, atol=1e-12)


def test_worked_storage_example():
    rows = [ln.split() for ln in open(os.path.join(GOLDEN, "polarquant_storage_example.txt"))
            if ln.strip() and not ln.startswith("#")]
    levels = [(int(a), int(b), int(c)) for a, b, c in (r for r in rows if r[0].isdigit())]
    extra = {r[0]: r[1:] for r in rows if not r[0].isdigit()}
    assert tuple(b for _, _, b in levels) == polar.LEVEL_BITS_D128
    assert [n for _, n, _ in levels] == [D >> lv for lv, _, _ in levels]  # d / 2^l angles at level l
    assert extra["radii"] == ["8", str(polar.RADIUS_BITS)]
    assert polar.bits_per_vector(D) == int(extra["total"][0])
    assert round(16 * D / polar.bits_per_vector(D), 2) == float(extra["ratio"][0])
    # the oracle packs each level's angle bits into ceil(bits / 32) words
    q = polar.quantize(np.random.default_rng(0).standard_normal((3, D)), params.rotation(D, 2), polar.codebooks())
    assert [w.shape[1] for w in q["words"]] == [-(-n * b // 32) for _, n, b in levels]


@pytest.mark.parametrize("level", [2, 3, 4, 5, 8])
def test_density_constant_against_adaptive_quadrature(level):
    k = polar.level_dim(level)
    mass = integrate.quad(lambda t: np.sin(2 * t) ** (k - 1), 0, np.pi / 2, epsabs=1e-14, epsrel=1e-13)[0]
    total = integrate.quad(lambda t: float(polar.angle_density(t, level)), 0, np.pi / 2, epsabs=1e-14,
                           epsrel=1e-13)[0]
    assert abs(total - 1.0) < 1e-12
    # the page's constant Gamma(k) / (2^(k-2) Gamma(k/2)^2) is 1 / mass
    assert float(polar.angle_density(np.pi / 4, level)) == pytest.approx(1.0 / mass, rel=1e-12)
    mean = integrate.quad(lambda t: t * float(polar.angle_density(t, level)), 0, np.pi / 2, epsabs=1e-14)[0]
    assert mean == pytest.approx(np.pi / 4, abs=1e-12)  # E[Theta] = pi / 4


@pytest.mark.parametrize("level", [2, 3, 4, 6])
def test_angle_cdf_is_the_incomplete_beta(level):
    # u = sin^2(theta) of the lemma's density is Beta(k/2, k/2): P(Theta <= t) = I_{sin^2 t}(k/2, k/2)
    from scipy.special import betainc

    k = polar.level_dim(level)
    for t in (0.05, 0.3, 0.6, np.pi / 4, 1.0, 1.4):
        cdf = integrate.quad(lambda u: float(polar.angle_density(u, level)), 0, t, epsabs=1e-15, epsrel=1e-13,
                             limit=200)[0]
        assert cdf == pytest.approx(betainc(k / 2, k / 2, np.sin(t) ** 2), abs=1e-12)


@pytest.mark.parametrize("level", [2, 3, 4])
def test_density_matches_gaussian_subvector_angles(level):
    k = polar.level_dim(level)
    g = np.random.default_rng(level).standard_normal((200000, 2, k))
    th = np.arctan2(np.linalg.norm(g[:, 1], axis=1), np.linalg.norm(g[:, 0], axis=1))
    grid = np.linspace(0, np.pi / 2, 41)[1:-1]
    cdf = np.array([integrate.quad(lambda t: float(polar.angle_density(t, level)), 0, u)[0] for u in grid])
    emp = (th[:, None] <= grid[None, :]).mean(axis=0)
    assert np.abs(emp - cdf).max() < 4e-3  # about 3.5 standard errors at 2e5 samples


def test_level1_codebook_is_the_uniform_closed_form():
    c, it = polar.lloyd_max_angles(1, 4)
    np.testing.assert_allclose(c, (2 * np.arange(16) + 1) * np.pi / 16, rtol=0, atol=1e-14)
    assert it <= 2


@pytest.mark.parametrize("level,bits", [(2, 2), (3, 2), (4, 2), (2, 3), (4, 4)])
def test_angle_codebooks(level, bits):
    c, _ = polar.lloyd_max_angles(level, bits)
    K = 1 << bits
    # symmetric about pi/4 (the density is)
    np.testing.assert_allclose(c + c[::-1], np.full(K, np.pi / 2), atol=1e-12)
    # each centroid is the density-weighted mean of its cell (adaptive quadrature, independent of the
    # oracle's Gauss-Legendre rule), and lies between its cell's midpoint and pi/4 ("the centroids move
    # towards the peak of the distribution, not the geometric centre of the bin")
    edges = np.concatenate([[0.0], 0.5 * (c[:-1] + c[1:]), [np.pi / 2]])
    f = lambda t: float(polar.angle_density(t, level))
    for i in range(K):
        m0 = integrate.quad(f, edges[i], edges[i + 1], epsabs=1e-15, epsrel=1e-13)[0]
        m1 = integrate.quad(lambda t: t * f(t), edges[i], edges[i + 1], epsabs=1e-15, epsrel=1e-13)[0]
        assert c[i] == pytest.approx(m1 / m0, abs=1e-11)
        mid = 0.5 * (edges[i] + edges[i + 1])
        assert abs(c[i] - np.pi / 4) <= abs(mid - np.pi / 4) + 1e-15


def test_quantize_roundtrip_errors_and_zero_vector():
    Pi = params.rotation(D, 2)
    books = polar.codebooks()
    x = np.random.default_rng(3).standard_normal((400, D))
    x[7] = 0.0
    q = polar.quantize(x, Pi, books)
    # level-1 angles: the 16 cells have width pi/8, so the angle error is at most pi/16
    th_hat = books[0][q["codes"][0]]
    assert np.abs(th_hat - q["angles"][0]).max() <= np.pi / 16 + 1e-12
    # packed words hold every level's codes (LSB first) and nothing else
    assert [w.shape[1] for w in q["words"]] == [8, 2, 1, 1]
    xh = polar.dequantize(q, Pi, books)
    assert np.all(xh[7] == 0.0)
    keep = np.arange(400) != 7
    rel = np.linalg.norm(xh[keep] - x[keep], axis=1) / np.linalg.norm(x[keep], axis=1)
    # with exact angles the only error is the fp16 radii (relative 2^-11); quantized angles dominate
    exact = polar.inverse_polar(q["angles"], q["radii"]) @ Pi
    rel_exact = np.linalg.norm(exact[keep] - x[keep], axis=1) / np.linalg.norm(x[keep], axis=1)
    assert rel_exact.max() < 2.0 ** -11
    assert 0.05 < rel.mean() < 0.5
    # more bits per level never hurt on average
    books_hi = polar.codebooks((5, 3, 3, 3))
    xh_hi = polar.dequantize(polar.quantize(x, Pi, books_hi, (5, 3, 3, 3)), Pi, books_hi)
    rel_hi = np.linalg.norm(xh_hi[keep] - x[keep], axis=1) / np.linalg.norm(x[keep], axis=1)
    assert rel_hi.mean() < rel.mean()
