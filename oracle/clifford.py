"""Cl(3,0) geometric algebra, written out from its definition.

"TurboQuant + RotorQuant", section "How RotorQuant Works": multivectors have 8
components in the basis order [1, e1, e2, e3, e12, e13, e23, e123]; a rotor has
the 4 nonzero components [s, 0, 0, 0, b12, b13, b23, 0]; a vector v is rotated
by the sandwich v' = R v R~. Section "Non-Commutative Algebra Bug Fix": the
sandwich is (R * v) * R~ -- rotor on the left, then the reversed rotor on the
right -- and the wrong order R~ * (R * v) is a known bug.

The product here is the generic 8x8 blade product (no sparsity is exploited):
each basis blade is the ordered tuple of its vector indices, two blades are
multiplied by concatenating the tuples and sorting them with adjacent swaps,
each swap of two different vectors flips the sign (e_i e_j = -e_j e_i), and
each adjacent equal pair cancels (e_i e_i = +1 in Cl(3,0)).
"""

import numpy as np

# Basis blades in the order the README gives: 1, e1, e2, e3, e12, e13, e23, e123.
BLADES = [(), (1,), (2,), (3,), (1, 2), (1, 3), (2, 3), (1, 2, 3)]
GRADE = np.array([len(b) for b in BLADES])


def _blade_product(a, b):
    """Product of two basis blades: returns (sign, blade tuple)."""
    seq = list(a) + list(b)
    sign = 1
    # bubble sort with adjacent swaps; each swap of distinct vectors anticommutes
    changed = True
    while changed:
        changed = False
        for i in range(len(seq) - 1):
            if seq[i] > seq[i + 1]:
                seq[i], seq[i + 1] = seq[i + 1], seq[i]
                sign = -sign
                changed = True
    # cancel equal neighbours: e_i e_i = +1
    out = []
    for v in seq:
        if out and out[-1] == v:
            out.pop()
        else:
            out.append(v)
    return sign, tuple(out)


def product_table():
    """sign[i, j] and index[i, j] with blade_i * blade_j = sign * blade_index."""
    sign = np.zeros((8, 8), dtype=np.int64)
    index = np.zeros((8, 8), dtype=np.int64)
    for i, a in enumerate(BLADES):
        for j, b in enumerate(BLADES):
            s, blade = _blade_product(a, b)
            sign[i, j] = s
            index[i, j] = BLADES.index(blade)
    return sign, index


_SIGN, _INDEX = product_table()


def gp(a, b):
    """Geometric product of multivectors a, b with shape [..., 8] (float64)."""
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    shape = np.broadcast_shapes(a.shape, b.shape)
    out = np.zeros(shape, dtype=np.float64)
    for i in range(8):
        for j in range(8):
            out[..., _INDEX[i, j]] += _SIGN[i, j] * a[..., i] * b[..., j]
    return out


def reverse(a):
    """Reversion a~: a blade of grade k changes sign by (-1)^(k(k-1)/2)."""
    a = np.asarray(a, dtype=np.float64)
    s = np.array([(-1) ** (k * (k - 1) // 2) for k in GRADE], dtype=np.float64)
    return a * s


def embed_vector(v):
    """Grade-1 multivector from 3-vectors v[..., 3] (components on e1, e2, e3)."""
    v = np.asarray(v, dtype=np.float64)
    out = np.zeros(v.shape[:-1] + (8,), dtype=np.float64)
    out[..., 1:4] = v
    return out


def rotor(s, b12, b13, b23):
    """Rotor multivector [s, 0, 0, 0, b12, b13, b23, 0] from its 4 components."""
    s = np.asarray(s, dtype=np.float64)
    out = np.zeros(s.shape + (8,), dtype=np.float64)
    out[..., 0] = s
    out[..., 4] = b12
    out[..., 5] = b13
    out[..., 6] = b23
    return out


def sandwich(R, v):
    """Forward sandwich v' = (R v) R~ of vector(s) v[..., 3]; returns the full
    multivector [..., 8] (its non-vector grades are zero for a rotor R)."""
    return gp(gp(R, embed_vector(v)), reverse(R))


def unsandwich(R, v):
    """Inverse sandwich v = (R~ v') R, used by dequantization."""
    return gp(gp(reverse(R), embed_vector(v)), R)
