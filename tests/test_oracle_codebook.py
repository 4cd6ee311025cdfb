"""Pins for the oracle's Lloyd-Max codebook (CPU only)."""

import math
import os

import numpy as np
import pytest
from scipy import integrate, special

from oracle import codebook

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rows(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return [ln.split() for ln in f if ln.strip() and not ln.startswith("#")]


@pytest.mark.parametrize("d", [2, 3, 5, 128, 1536])
def test_density_integrals_against_quadrature(d):
    f = lambda x: float(codebook.density(x, d))
    pts = [-1.0, -0.3, 0.0, 0.05, 0.4, 1.0]
    # quadrature of the density itself is an independent route to the closed forms
    total, _ = integrate.quad(f, -1, 1, points=[0.0], limit=200)
    assert abs(total - 1.0) < 1e-8
    second, _ = integrate.quad(lambda x: x * x * f(x), -1, 1, points=[0.0], limit=200)
    assert abs(second - 1.0 / d) < 1e-8
    for a, b in zip(pts[:-1], pts[1:]):
        m0, _ = integrate.quad(f, a, b, limit=200)
        m1, _ = integrate.quad(lambda x: x * f(x), a, b, limit=200)
        assert abs(codebook.cell_mass(a, b, d) - m0) < 1e-9
        assert abs(codebook.cell_first_moment(a, b, d) - m1) < 1e-9


def test_density_matches_sphere_coordinate_samples():
    # a coordinate of a uniform unit vector (normalised Gaussian) has this law
    g = np.random.default_rng(0)
    d = 20
    x = g.normal(size=(200000, d))
    c1 = x[:, 0] / np.linalg.norm(x, axis=1)
    for t in (-0.5, -0.1, 0.0, 0.2, 0.45):
        emp = np.mean(c1 <= t)
        assert abs(emp - codebook.cdf(t, d)) < 5 * math.sqrt(0.25 / c1.size)


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_d3_is_uniform_and_centroids_are_closed_form(bits):
    # d = 3: f(x) = 1/2 on [-1, 1], so the optimum is the uniform quantizer
    c, t, _ = codebook.lloyd_max(3, bits)
    K = 2 ** bits
    expect = -1.0 + (2.0 * np.arange(K) + 1.0) / K
    assert np.abs(c - expect).max() < 1e-12
    assert abs(codebook.distortion(c, 3) - (2.0 / K) ** 2 / 12.0) < 1e-14


@pytest.mark.parametrize("d", [4, 8, 128, 1536])
def test_one_bit_centroid_is_mean_abs_coordinate(d):
    c, t, _ = codebook.lloyd_max(d, 1)
    e_abs = math.exp(special.gammaln(d / 2) - special.gammaln((d + 1) / 2)) / math.sqrt(math.pi)
    assert abs(c[1] - e_abs) < 1e-13 and abs(c[0] + e_abs) < 1e-13
    assert t[0] == pytest.approx(0.0, abs=1e-15)
    if d == 128:
        assert round(c[1] * math.sqrt(d), 5) == 0.79944


@pytest.mark.parametrize("d,bits", [(16, 3), (128, 2), (128, 3), (128, 4), (1536, 4)])
def test_lloyd_fixed_point_symmetry_and_local_optimality(d, bits):
    c, t, it = codebook.lloyd_max(d, bits)
    assert np.all(np.diff(c) > 0)
    assert np.abs(c + c[::-1]).max() < 1e-12
    assert np.abs(t - 0.5 * (c[:-1] + c[1:])).max() == 0.0
    # each centroid is the conditional mean of its cell (checked by quadrature)
    f = lambda x: float(codebook.density(x, d))
    edges = np.concatenate([[-1.0], t, [1.0]])
    for k in range(len(c)):
        m0, _ = integrate.quad(f, edges[k], edges[k + 1], limit=200)
        m1, _ = integrate.quad(lambda x: x * f(x), edges[k], edges[k + 1], limit=200)
        assert abs(m1 / m0 - c[k]) < 1e-9
    # moving any centroid raises the distortion
    D = codebook.distortion(c, d)
    for k in range(len(c)):
        for eps in (1e-3, -1e-3):
            cp = c.copy()
            cp[k] += eps / math.sqrt(d)
            assert codebook.distortion(np.sort(cp), d) > D


def test_any_start_converges_to_the_same_codebook():
    # f is log-concave, so Lloyd's fixed point is unique
    c_ref, _, _ = codebook.lloyd_max(64, 3)
    d, K = 64, 8
    c = np.linspace(-0.9, 0.9, K)
    for _ in range(20000):
        t = 0.5 * (c[:-1] + c[1:])
        lo = np.concatenate([[-1.0], t])
        hi = np.concatenate([t, [1.0]])
        c_new = codebook.cell_first_moment(lo, hi, d) / codebook.cell_mass(lo, hi, d)
        if np.abs(c_new - c).max() < 1e-14:
            break
        c = c_new
    assert np.abs(c - c_ref).max() < 1e-11


def test_pages_mse_table_d128():
    # the analytic unit-vector MSE d * D rounds to the README's printed values
    for bits, tq_mse, rq_mse, _cos in _rows("mse_quality_table.txt"):
        c, _, _ = codebook.lloyd_max(128, int(bits))
        total = 128 * codebook.distortion(c, 128)
        assert round(total, 3) == pytest.approx(float(tq_mse), abs=1e-12)
        assert round(total, 3) == pytest.approx(float(rq_mse), abs=1e-12)


def test_large_d_limit_is_max_1960_gaussian_quantizer():
    for row in _rows("max1960_gaussian_levels.txt"):
        K, mse, levels = int(row[0]), float(row[1]), np.array([float(v) for v in row[2:]])
        c, _, _ = codebook.lloyd_max(4096, int(math.log2(K)))
        pos = c[K // 2:] * math.sqrt(4096)
        assert np.abs(pos / levels - 1).max() < 3e-3
        assert abs(4096 * codebook.distortion(c, 4096) / mse - 1) < 3e-3


def test_theorem1_constants_and_bound_reading():
    consts = {r[0]: (float(r[1]), float(r[2])) for r in _rows("theorem1_constants.txt")}
    d = 1536
    scaled = []
    for bits in (1, 2, 3, 4, 5):
        c, _, _ = codebook.lloyd_max(d, bits)
        scaled.append(d * codebook.distortion(c, d) * 4.0 ** bits)
    b1, tol1 = consts["b1_constant"]
    assert abs(scaled[0] - b1) < tol1
    # D * 4^b grows with b toward sqrt(3) pi / 2 (the Panter-Dite constant)
    assert all(a < b for a, b in zip(scaled, scaled[1:]))
    limit, tol = consts["large_b_constant"]
    assert abs(math.sqrt(3) * math.pi / 2 - limit) < tol
    assert scaled[-1] < math.sqrt(3) * math.pi / 2
    # Theorem 1 bound under the reading sqrt(3) pi / 2: holds for every b at d = 128
    for bits in (1, 2, 3, 4):
        c, _, _ = codebook.lloyd_max(128, bits)
        total = 128 * codebook.distortion(c, 128)
        assert total <= math.sqrt(3) * math.pi / 2 * 4.0 ** -bits
        # the literal sqrt(3 pi)/2 ~ 1.53 is violated already at b = 2 (the
        # extraction garbled the constant)
        if bits >= 2:
            assert total > math.sqrt(3 * math.pi) / 2 * 4.0 ** -bits


def test_rejects_degenerate_dimension():
    with pytest.raises(ValueError):
        codebook.lloyd_max(1, 2)
