"""The method's random parameters, drawn from the counter-based streams of ``rng``.

* Rotors -- "TurboQuant + RotorQuant", section "How RotorQuant Works": d is cut
  into groups of 3 coordinates, each rotated by its own rotor with 4 nonzero
  components (s, b12, b13, b23). The pages say only "random unit rotors"; the
  plain reading taken here is the uniform distribution on the unit 3-sphere:
  4 i.i.d. N(0,1) draws, divided by their Euclidean norm.
* Pi -- "TurboQuant 论文解读", section "随机旋转（Lemma 1）" and its demo: a random
  orthogonal matrix from the QR decomposition of a d x d Gaussian matrix. The
  column signs are fixed so that diag(R) > 0, which makes Pi unique for a given
  Gaussian matrix (and Haar distributed).
* T -- same blog, section "QJL 内积无偏估计（Theorem 2）": the QJL projection has
  i.i.d. N(0,1) entries; T is m x d with m = d in the demo.

Stream layout: entry (i, j) of a row-major r x c matrix is normal number i*c + j
of its stream; rotor g takes normals 4g .. 4g+3 in the order s, b12, b13, b23.
"""

import numpy as np

from . import rng


def n_groups(d):
    """G = ceil(d / 3) rotor groups ("4 per group x ceil(d/3)" parameters)."""
    return -(-d // 3)


def rotors(d, seed):
    """[G, 4] unit rotors (s, b12, b13, b23), float64."""
    G = n_groups(d)
    r = rng.normals(seed, 4 * G).reshape(G, 4)
    return r / np.linalg.norm(r, axis=1, keepdims=True)


def rotation(d, seed):
    """[d, d] orthogonal Pi = Q diag(sign(diag R)) with Q R = Gaussian matrix."""
    a = rng.normals(seed, d * d).reshape(d, d)
    q, r = np.linalg.qr(a)
    return q * np.sign(np.diag(r))[None, :]


def qjl_matrix(m, d, seed):
    """[m, d] matrix of i.i.d. N(0, 1) entries."""
    return rng.normals(seed, m * d).reshape(m, d)
