"""PolarQuant: random preconditioning, recursive polar transform, per-level angle codebooks.

TEST INFRASTRUCTURE ONLY (see the package docstring).

"TurboQuant и PolarQuant: математика квантизации KV-кэша в LLM":
* "Факт 1" / "Шаг 1: предобусловливание": the vector is first multiplied by a
  fixed random orthogonal matrix (here Pi of params.rotation, the same family
  as the page's Gram-Schmidt of a Gaussian matrix).
* "Полярное преобразование" / "Шаг 2": level 1 pairs consecutive coordinates
  (a, b) = (y_2i, y_2i+1) into a radius sqrt(a^2 + b^2) and an angle
  atan2(b, a) taken in [0, 2 pi); every further level pairs consecutive radii
  of the level below the same way, and since radii are >= 0 its angles lie in
  [0, pi/2]. The angles of every level are stored; the radii of the last level
  are kept as 16-bit floats.
* The lemma quoted there: at a level whose radii are norms of k-dimensional
  Gaussian sub-vectors, the angle has density
  Gamma(k) / (2^(k-2) Gamma(k/2)^2) * sin^(k-1)(2 theta) on [0, pi/2].
  A level-l radius (l >= 1) is the norm of 2^l consecutive coordinates, so the
  angles of level l >= 2 have k = 2^(l-1); level 1 angles are uniform on
  [0, 2 pi). Angles do not depend on the scale of y, so the same densities hold
  for a rotated fixed vector, which is a uniformly random direction times its
  norm.
* "Шаг 3: построение кодовых книг": one Lloyd-Max codebook per level for that
  density (boundaries at midpoints of neighbouring centroids, centroids the
  density-weighted means of their cells, repeated to convergence); quantize to
  the nearest centroid.
* "Степень сжатия": at d = 128, four levels with 4, 2, 2, 2 bits and 8 radii
  of 16 bits, 496 bits per vector.

Readings: the worked example fixes the level count and the bits (4 levels,
(4, 2, 2, 2) bits at d = 128); the level-1 codebook is Lloyd on the interval
[0, 2 pi) with the uniform density; ties go to the lower index; a zero pair
has angle atan2(0, 0) = 0.
"""

import numpy as np
from scipy.special import gammaln

from . import codes as codes_mod

LEVEL_BITS_D128 = (4, 2, 2, 2)
RADIUS_BITS = 16

_GL_X, _GL_W = np.polynomial.legendre.leggauss(64)  # Gauss-Legendre nodes on [-1, 1]


def level_dim(level):
    """k: the dimension of the sub-vectors whose norms form the pairs of `level` (1-based)."""
    return 1 << (level - 1)


def angle_range(level):
    return (0.0, 2.0 * np.pi) if level == 1 else (0.0, 0.5 * np.pi)


def angle_density(theta, level):
    """Density of the level's angles on its range (uniform for level 1)."""
    theta = np.asarray(theta, dtype=np.float64)
    if level == 1:
        return np.full_like(theta, 1.0 / (2.0 * np.pi))
    k = level_dim(level)
    log_c = gammaln(k) - (k - 2) * np.log(2.0) - 2.0 * gammaln(k / 2.0)
    return np.exp(log_c) * np.sin(2.0 * theta) ** (k - 1)


def _cell_moments(a, b, level):
    """(mass, first moment) of every cell [a_i, b_i] by 64-point Gauss-Legendre quadrature."""
    a = np.asarray(a, dtype=np.float64)[:, None]
    b = np.asarray(b, dtype=np.float64)[:, None]
    t = 0.5 * (b - a) * _GL_X[None, :] + 0.5 * (a + b)
    w = 0.5 * (b - a) * _GL_W[None, :]
    f = angle_density(t, level)
    return (w * f).sum(axis=1), (w * f * t).sum(axis=1)


def lloyd_max_angles(level, bits, tol=1e-13, max_iter=200000):
    """Centroids (ascending) of the level's angle codebook; returns (centroids, iterations)."""
    lo, hi = angle_range(level)
    K = 1 << bits
    c = lo + (np.arange(K) + 0.5) * (hi - lo) / K
    for it in range(1, max_iter + 1):
        edges = np.concatenate([[lo], 0.5 * (c[:-1] + c[1:]), [hi]])
        mass, mom = _cell_moments(edges[:-1], edges[1:], level)
        c_new = mom / mass
        delta = np.abs(c_new - c).max()
        c = c_new
        if delta < tol:
            return c, it
    raise RuntimeError("Lloyd iteration did not converge")


def polar_transform(y, n_levels):
    """y [N, d] -> (angles: list of n_levels arrays [N, d / 2^l], radii [N, d / 2^n_levels])."""
    r = np.asarray(y, dtype=np.float64)
    angles = []
    for level in range(1, n_levels + 1):
        a, b = r[:, 0::2], r[:, 1::2]
        th = np.arctan2(b, a)
        if level == 1:
            th = np.mod(th, 2.0 * np.pi)
        angles.append(th)
        r = np.sqrt(a * a + b * b)
    return angles, r


def inverse_polar(angles, radii):
    """Undo polar_transform: from the last level's radii down to the coordinates."""
    r = np.asarray(radii, dtype=np.float64)
    for th in reversed(angles):
        out = np.empty((r.shape[0], 2 * r.shape[1]))
        out[:, 0::2] = r * np.cos(th)
        out[:, 1::2] = r * np.sin(th)
        r = out
    return r


def codebooks(level_bits=LEVEL_BITS_D128):
    return [lloyd_max_angles(level, b)[0] for level, b in enumerate(level_bits, start=1)]


def quantize(x, Pi, books, level_bits=LEVEL_BITS_D128):
    """x [N, d] -> dict(codes: per-level code arrays, words: per-level packed words, radii fp16 values)."""
    y = np.asarray(x, dtype=np.float64) @ np.asarray(Pi, dtype=np.float64).T
    angles, radii = polar_transform(y, len(level_bits))
    codes = [codes_mod.nearest(th, c) for th, c in zip(angles, books)]
    words = [codes_mod.pack(cd, b) for cd, b in zip(codes, level_bits)]
    return {"codes": codes, "words": words, "radii": radii.astype(np.float16).astype(np.float64),
            "angles": angles}


def dequantize(q, Pi, books):
    """x_hat [N, d] from the per-level codes and the 16-bit radii."""
    th_hat = [np.asarray(c, dtype=np.float64)[cd] for cd, c in zip(q["codes"], books)]
    y_hat = inverse_polar(th_hat, q["radii"])
    return y_hat @ np.asarray(Pi, dtype=np.float64)


def bits_per_vector(d, level_bits=LEVEL_BITS_D128, radius_bits=RADIUS_BITS):
    """Stored bits of one vector: every level's angle codes plus the last level's radii."""
    total, n = 0, d
    for b in level_bits:
        n //= 2
        total += n * b
    return total + n * radius_bits
