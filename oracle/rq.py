"""RotorQuant quantize / dequantize, step by step.

"TurboQuant + RotorQuant":
* "Codebook Calibration Fix", item 2 (norm separation): every vector is divided
  by its L2 norm before quantization, the norm is stored separately, and the
  reconstruction is multiplied by it.
* "How RotorQuant Works": the (unit) vector is cut into groups of 3 coordinates
  (d = 128 gives 43 groups; the last group is zero-padded) and each group is
  rotated by its own rotor with the sandwich v' = R v R~.
* "The Fused CUDA Kernel": embed (3 dims -> multivector) -> R x R~ -> Lloyd-Max
  quantize -> R~ x R -> extract.
* Section "Codebook Calibration Fix", item 1: one Lloyd-Max codebook built for
  d_eff = d quantizes the rotated vector-grade coordinates.

Reading taken where the pages are silent: the 3G rotated coordinates, the
rotated pad coordinate included, are each quantized with that one codebook and
stored (3G codes per vector, 129 at d = 128); extraction after the inverse
sandwich drops coordinates >= d. A zero vector stores norm 0 and reconstructs
to 0; its codes are those of y = 0.
"""

import numpy as np

from . import clifford, codes as codes_mod
from .params import n_groups


def split_norm(x):
    """(norms [N], u [N, d]) with u = x / ||x|| and u = 0 for a zero row."""
    x = np.asarray(x, dtype=np.float64)
    n = np.sqrt(np.sum(x * x, axis=1))
    safe = np.where(n > 0, n, 1.0)
    return n, np.where(n[:, None] > 0, x / safe[:, None], 0.0)


def _rotor_mv(rotors):
    r = np.asarray(rotors, dtype=np.float64)
    return clifford.rotor(r[:, 0], r[:, 1], r[:, 2], r[:, 3])  # [G, 8]


def rotate(u, rotors):
    """Forward sandwich of every 3-group: u [N, d] -> y [N, 3G] (pad rotated too)."""
    N, d = u.shape
    G = n_groups(d)
    v = np.zeros((N, 3 * G))
    v[:, :d] = u
    out = clifford.sandwich(_rotor_mv(rotors)[None, :, :], v.reshape(N, G, 3))
    other = np.abs(out[..., [0, 4, 5, 6, 7]]).max() if out.size else 0.0
    assert other < 1e-12, "rotor sandwich produced non-vector grades"
    return out[..., 1:4].reshape(N, 3 * G)


def unrotate(y, rotors, d):
    """Inverse sandwich of every 3-group, then drop the pad: [N, 3G] -> [N, d]."""
    N = y.shape[0]
    G = n_groups(d)
    out = clifford.unsandwich(_rotor_mv(rotors)[None, :, :], np.asarray(y).reshape(N, G, 3))
    other = np.abs(out[..., [0, 4, 5, 6, 7]]).max() if out.size else 0.0
    assert other < 1e-12, "inverse sandwich produced non-vector grades"
    return out[..., 1:4].reshape(N, 3 * G)[:, :d]


def quantize(x, rotors, centroids, bits):
    """x [N, d] -> dict(words [N, W] uint32, codes [N, 3G], norms [N], y [N, 3G])."""
    n, u = split_norm(x)
    y = rotate(u, rotors)
    idx = codes_mod.nearest(y, centroids)
    return {"words": codes_mod.pack(idx, bits), "codes": idx, "norms": n, "y": y}


def dequantize(words, norms, rotors, centroids, bits, d):
    """Packed words [N, W] + norms [N] -> x_hat [N, d]."""
    G = n_groups(d)
    idx = codes_mod.unpack(words, 3 * G, bits)
    c_hat = np.asarray(centroids, dtype=np.float64)[idx]
    return np.asarray(norms, dtype=np.float64)[:, None] * unrotate(c_hat, rotors, d)


def roundtrip(x, rotors, centroids, bits):
    """Quantize then dequantize; returns the quantize dict plus 'xhat'."""
    q = quantize(x, rotors, centroids, bits)
    q["xhat"] = dequantize(q["words"], q["norms"], rotors, centroids, bits, np.asarray(x).shape[1])
    return q
