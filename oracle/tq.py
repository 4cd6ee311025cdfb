"""TurboQuant-mse (Algorithm 1) and TurboQuant-prod (Algorithm 2).

* arXiv 2504.19874 summary page, "方法": Algorithm 1 multiplies x by a random
  rotation Pi, maps every rotated coordinate to its nearest precomputed
  Lloyd-Max centroid, and dequantizes by looking the centroids up and applying
  Pi^T. Algorithm 2 runs the MSE quantizer at b-1 bits, takes the residual,
  and stores a 1-bit QJL sketch (signs of a Gaussian projection) of it; the
  reconstruction adds the scaled QJL reconstruction to the MSE one.
* "TurboQuant 论文解读", "随机旋转（Lemma 1）": y = Pi x, and Pi^-1 = Pi^T
  undoes it. "QJL 内积无偏估计（Theorem 2）": r = x - x_mse, qjl = sign(S r),
  x_qjl = scale * ||r|| * S^T qjl, x = x_mse + x_qjl.
* "TurboQuant + RotorQuant", "How TurboQuant Works": the estimator is
  <q, k> ~ <q, k_mse> + ||r|| * sqrt(pi/2) / m * <S q, sign(S r)>, i.e. the QJL
  scale is sqrt(pi/2) / m (the demo uses the same, with m = d). The blog's
  sqrt((pi/2)/d) is read as a formula garbled in extraction.
* Norm separation ("Codebook Calibration Fix", item 2) as for RotorQuant.

Readings where the pages leave a step open:
* sign(0) := +1 (a 1-bit sign cannot hold the 0 of numpy's sign). Bit j of the
  sketch is 1 for +1 and 0 for -1, packed LSB first, m/32 words per row.
* S := T Pi with T an m x d i.i.d. N(0,1) matrix. S is then itself i.i.d.
  N(0,1). The residual is formed in rotated coordinates, r_rot = y - c_hat;
  with an orthogonal Pi this is exactly Pi r, ||r_rot|| = ||r|| and
  S r = T r_rot, so the stored gamma and signs are the pages' quantities.
  ``prod_quantize_literal`` writes the pages' form out for comparison.
* The sign decision is taken on the float64 product T r_rot itself: no
  rounding of any implementation's operands enters the oracle.
"""

import numpy as np

from . import codes as codes_mod
from .rq import split_norm

QJL_SCALE_NUM = np.sqrt(np.pi / 2.0)  # the estimator's sqrt(pi/2); divided by m


def mse_quantize(x, Pi, centroids, bits):
    """Algorithm 1 quantize: x [N, d] -> dict(words, codes, norms, y)."""
    n, u = split_norm(x)
    Pi = np.asarray(Pi, dtype=np.float64)
    y = u @ Pi.T  # y = Pi u for every row
    idx = codes_mod.nearest(y, centroids)
    return {"words": codes_mod.pack(idx, bits), "codes": idx, "norms": n, "y": y}


def mse_dequantize(words, norms, Pi, centroids, bits, d):
    """Algorithm 1 dequantize: x_hat = ||x|| * Pi^T c_hat."""
    idx = codes_mod.unpack(words, d, bits)
    c_hat = np.asarray(centroids, dtype=np.float64)[idx]
    return np.asarray(norms, dtype=np.float64)[:, None] * (c_hat @ np.asarray(Pi, dtype=np.float64))


def _sign_bits(p):
    """sign with sign(0) = +1, as bits: 1 for +1, 0 for -1."""
    return (p >= 0).astype(np.int64)


def prod_quantize(x, Pi, T, centroids_mse, bits):
    """Algorithm 2 quantize with b = ``bits`` total (b-1 MSE bits + 1 QJL bit).

    Returns dict(words (MSE codes, b-1 bits), codes, signs_words [N, m/32],
    signs (+1/-1) [N, m], gammas [N], norms [N], y, r_rot [N, d], p [N, m],
    z [N, m]) where p = T r_rot row by row (the sketch's decision value:
    sign bit j is p[:, j] >= 0) and z[:, j] is the cosine between row j of T
    and the residual."""
    n, u = split_norm(x)
    Pi = np.asarray(Pi, dtype=np.float64)
    T = np.asarray(T, dtype=np.float64)
    y = u @ Pi.T
    idx = codes_mod.nearest(y, centroids_mse)
    c_hat = np.asarray(centroids_mse, dtype=np.float64)[idx]
    r_rot = y - c_hat
    gamma = np.sqrt(np.sum(r_rot * r_rot, axis=1))
    p = r_rot @ T.T  # T r_rot, row by row
    bits_s = _sign_bits(p)
    t_norm = np.linalg.norm(T, axis=1)
    z = p / (t_norm[None, :] * np.where(gamma > 0, gamma, 1.0)[:, None])
    return {
        "words": codes_mod.pack(idx, bits - 1),
        "codes": idx,
        "signs_words": codes_mod.pack(bits_s, 1),
        "signs": 2 * bits_s - 1,
        "gammas": gamma,
        "norms": n,
        "y": y,
        "r_rot": r_rot,
        "p": p,
        "z": z,
    }


def prod_dequantize(words, signs_words, gammas, norms, Pi, T, centroids_mse, bits, d):
    """x_hat = ||x|| * Pi^T (c_hat + sqrt(pi/2)/m * gamma * T^T s)."""
    T = np.asarray(T, dtype=np.float64)
    m = T.shape[0]
    idx = codes_mod.unpack(words, d, bits - 1)
    c_hat = np.asarray(centroids_mse, dtype=np.float64)[idx]
    s = 2 * codes_mod.unpack(signs_words, m, 1) - 1
    g = np.asarray(gammas, dtype=np.float64)
    w = c_hat + (QJL_SCALE_NUM / m) * g[:, None] * (s @ T)
    return np.asarray(norms, dtype=np.float64)[:, None] * (w @ np.asarray(Pi, dtype=np.float64))


def qjl_sketch(r, T):
    """The QJL map on its own: signs_words = pack(sign(T r)), gammas = ||r||."""
    r = np.asarray(r, dtype=np.float64)
    p = r @ np.asarray(T, dtype=np.float64).T
    return {"signs_words": codes_mod.pack(_sign_bits(p), 1), "gammas": np.sqrt(np.sum(r * r, axis=1)), "p": p}


def prod_quantize_literal(x, Pi, T, centroids_mse):
    """The pages' form of Algorithm 2 on unit vectors, for comparison:
    x_mse = Pi^T c_hat, r = u - x_mse, qjl = sign(S r) with S = T Pi,
    x_tilde = x_mse + sqrt(pi/2)/m * ||r|| * S^T qjl. Returns (x_tilde, r, qjl)."""
    n, u = split_norm(x)
    Pi = np.asarray(Pi, dtype=np.float64)
    T = np.asarray(T, dtype=np.float64)
    S = T @ Pi
    m = T.shape[0]
    y = u @ Pi.T
    c_hat = np.asarray(centroids_mse, dtype=np.float64)[codes_mod.nearest(y, centroids_mse)]
    x_mse = c_hat @ Pi
    r = u - x_mse
    qjl = np.where(r @ S.T >= 0, 1.0, -1.0)
    x_tilde = x_mse + (QJL_SCALE_NUM / m) * np.linalg.norm(r, axis=1)[:, None] * (qjl @ S)
    return x_tilde, r, qjl
