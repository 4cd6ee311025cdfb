"""Lloyd-Max scalar codebook for one coordinate of a random unit vector.

"TurboQuant 论文解读", sections "Beta 分布" and "MSE 标量量化（Theorem 1）":
after a random rotation every coordinate of a unit vector in R^d has the same
known density, so the best 2^b reconstruction points can be computed offline
by minimising the expected squared error. For a uniform point on the sphere
S^(d-1) one coordinate has density

    f(x) = Gamma(d/2) / (sqrt(pi) Gamma((d-1)/2)) * (1 - x^2)^((d-3)/2),  -1 <= x <= 1.

"TurboQuant и PolarQuant" (paragraph on building the codebooks) gives Lloyd's
iteration: put each cell boundary half-way between neighbouring centroids,
then move each centroid to the probability-weighted mean of its cell, and
repeat until nothing moves.

"TurboQuant + RotorQuant", section "Codebook Calibration Fix": the codebook is
built with d_eff = d, the original vector dimension (also for RotorQuant).

Integrals are exact: with t = x^2, P(|X| <= a) = I_{a^2}(1/2, (d-1)/2) (the
regularized incomplete beta function, ``scipy.special.betainc``), and
int x (1-x^2)^k dx = -(1-x^2)^(k+1) / (2(k+1)) with k = (d-3)/2.
"""

import numpy as np
from scipy import special


def density_constant(d):
    """Normalising constant Gamma(d/2) / (sqrt(pi) Gamma((d-1)/2))."""
    return float(np.exp(special.gammaln(d / 2.0) - special.gammaln((d - 1) / 2.0)) / np.sqrt(np.pi))


def density(x, d):
    """f(x) for |x| <= 1 (zero outside)."""
    x = np.asarray(x, dtype=np.float64)
    inside = np.abs(x) <= 1.0
    xc = np.where(inside, x, 0.0)
    return np.where(inside, density_constant(d) * (1.0 - xc * xc) ** ((d - 3) / 2.0), 0.0)


def cdf(x, d):
    """F(x) = P(X <= x) = 1/2 + sign(x)/2 * I_{x^2}(1/2, (d-1)/2)."""
    x = np.clip(np.asarray(x, dtype=np.float64), -1.0, 1.0)
    return 0.5 + 0.5 * np.sign(x) * special.betainc(0.5, (d - 1) / 2.0, x * x)


def cell_mass(a, b, d):
    """int_a^b f(x) dx."""
    return cdf(b, d) - cdf(a, d)


def cell_first_moment(a, b, d):
    """int_a^b x f(x) dx, from the antiderivative -(1-x^2)^((d-1)/2) / (d-1)."""
    a = np.clip(np.asarray(a, dtype=np.float64), -1.0, 1.0)
    b = np.clip(np.asarray(b, dtype=np.float64), -1.0, 1.0)
    e = (d - 1) / 2.0
    return density_constant(d) * ((1.0 - a * a) ** e - (1.0 - b * b) ** e) / (2.0 * e)


def lloyd_max(d, bits, tol=1e-13, max_iter=100000):
    """Lloyd-Max centroids c[0..2^b) (ascending) and boundaries t[0..2^b-1).

    Returns (centroids, boundaries, iterations). Raises if not converged.
    The density is even, so the exact codebook is symmetric; the returned
    centroids are symmetrised, c_i = -c_(K-1-i) exactly, so that y = 0 lies
    exactly on the middle boundary for every even K.
    """
    if d < 2:
        raise ValueError("the coordinate density needs d >= 2")
    K = 2 ** bits
    # start from the distribution's (k + 1/2)/K quantiles
    q = (np.arange(K) + 0.5) / K
    c = np.sign(q - 0.5) * np.sqrt(special.betaincinv(0.5, (d - 1) / 2.0, np.abs(2 * q - 1)))
    for it in range(1, max_iter + 1):
        t = 0.5 * (c[:-1] + c[1:])
        lo = np.concatenate([[-1.0], t])
        hi = np.concatenate([t, [1.0]])
        c_new = cell_first_moment(lo, hi, d) / cell_mass(lo, hi, d)
        delta = np.max(np.abs(c_new - c))
        c = c_new
        if delta < tol:
            c = 0.5 * (c - c[::-1])
            return c, 0.5 * (c[:-1] + c[1:]), it
    raise RuntimeError("Lloyd-Max did not converge")


def distortion(centroids, d):
    """Per-coordinate MSE  sum_k int_cell_k (x - c_k)^2 f(x) dx  of the
    nearest-centroid quantizer (cells split at the midpoints).

    Uses E[X^2] = 1/d for a coordinate of a uniform unit vector."""
    c = np.asarray(centroids, dtype=np.float64)
    t = 0.5 * (c[:-1] + c[1:])
    lo = np.concatenate([[-1.0], t])
    hi = np.concatenate([t, [1.0]])
    m0 = cell_mass(lo, hi, d)
    m1 = cell_first_moment(lo, hi, d)
    return 1.0 / d - 2.0 * np.sum(c * m1) + np.sum(c * c * m0)
