"""RotorQuant in the pages' four-grade storage layout (172 indices per vector at d = 128).

TEST INFRASTRUCTURE ONLY (see the package docstring).

"TurboQuant + RotorQuant":
* "Parameter Efficiency": the RotorQuant parameters are the rotors plus four
  grade codebooks (scalar, vector, bivector, trivector).
* "FMA Count (d=128)" table: 172 stored indices per vector (TurboQuant: 128)
  and a 3-bit compression of 3.7x (TurboQuant: 4.9x).
* "The Fused CUDA Kernel": for a grade-1 input the sparse product has only
  vector and trivector outputs.

Reading taken: per group the stored indices are the three vector components
and the trivector component of the sandwiched multivector, 4 x 43 = 172 at
d = 128, each quantized with the codebook of its grade; the vector and
trivector codebooks are both the Lloyd-Max codebook of the rotated-coordinate
density (d_eff = d), the only one the pages define. The check that fixes the
reading: 172 codes of 3 bits are 64.5 bytes, with a 4-byte norm 256 / 69 B =
3.7x, the page's figure. For a unit rotor the trivector part of R v R~ is
identically zero, so its code is the code of exactly 0 (the lower middle code
by the tie rule); the inverse sandwich maps a pseudoscalar to itself, so the
extracted vector part, and x_hat, equal the three-component layout's.
"""

import numpy as np

from . import clifford, codes as codes_mod
from .params import n_groups
from .rq import split_norm

N_PER_GROUP = 4  # e1, e2, e3, e123


def quantize(x, rotors, centroids, bits):
    """x [N, d] -> dict(words [N, W] uint32 of 4G codes, codes [N, 4G], norms [N], mv [N, G, 8])."""
    n, u = split_norm(x)
    N, d = u.shape
    G = n_groups(d)
    v = np.zeros((N, 3 * G))
    v[:, :d] = u
    R = clifford.rotor(*np.asarray(rotors, dtype=np.float64).T)  # [G, 8]
    mv = clifford.sandwich(R[None, :, :], v.reshape(N, G, 3))  # [N, G, 8]
    # the trivector part is identically zero for a unit rotor; float64 leaves ~1e-17 of either
    # sign, which would pick either middle centroid, so it is stored as the code of exactly 0
    assert (np.abs(mv[..., 7]).max() if mv.size else 0.0) < 1e-12, "trivector part of a unit-rotor sandwich"
    tri = np.zeros(mv.shape[:-1] + (1,))
    comps = np.concatenate([mv[..., 1:4], tri], axis=2).reshape(N, N_PER_GROUP * G)
    idx = codes_mod.nearest(comps, centroids)
    return {"words": codes_mod.pack(idx, bits), "codes": idx, "norms": n, "mv": mv}


def dequantize(words, norms, rotors, centroids, bits, d):
    """Inverse sandwich of each group's (e1, e2, e3, e123) centroids; the vector part, pad dropped."""
    G = n_groups(d)
    N = np.asarray(words).shape[0]
    idx = codes_mod.unpack(words, N_PER_GROUP * G, bits).reshape(N, G, N_PER_GROUP)
    c = np.asarray(centroids, dtype=np.float64)[idx]
    mv = np.zeros((N, G, 8))
    mv[..., 1:4] = c[..., :3]
    mv[..., 7] = c[..., 3]
    R = clifford.rotor(*np.asarray(rotors, dtype=np.float64).T)
    out = clifford.gp(clifford.gp(clifford.reverse(R)[None], mv), R[None])  # R~ m R
    return np.asarray(norms, dtype=np.float64)[:, None] * out[..., 1:4].reshape(N, 3 * G)[:, :d]


def bytes_per_vector(d, bits, norm_bytes=4):
    """Storage of one vector: 4G codes of `bits` bits (as bytes, unrounded) plus the norm."""
    return N_PER_GROUP * n_groups(d) * bits / 8.0 + norm_bytes
