"""Pins for the oracle's random streams and Cl(3,0) algebra (CPU only)."""

import math
import os

import numpy as np
import pytest

from oracle import clifford, params, rng

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rows(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return [ln.split() for ln in f if ln.strip() and not ln.startswith("#")]


# ---------------------------------------------------------------- random streams

def test_splitmix64_reference_outputs():
    for idx, hexval in _rows("splitmix64_seed0.txt"):
        assert int(rng.splitmix64(0, [int(idx)])[0]) == int(hexval, 16)


def test_splitmix64_is_counter_based():
    # output i depends only on (seed, i): any subset of positions agrees
    full = rng.splitmix64(42, np.arange(100))
    some = rng.splitmix64(42, np.array([3, 99, 50]))
    assert list(some) == [full[3], full[99], full[50]]


def test_uniform_range_and_box_muller_moments():
    u = rng.uniform(5, np.arange(200000))
    assert u.min() > 0.0 and u.max() <= 1.0
    n = rng.normals(7, 400000)
    se = 1.0 / math.sqrt(n.size)
    assert abs(n.mean()) < 5 * se
    assert abs(n.var() - 1.0) < 5 * math.sqrt(2.0) * se
    assert abs((n ** 4).mean() - 3.0) < 5 * math.sqrt(96.0) * se
    # pairs are independent: correlation of even/odd members ~ 0
    assert abs(np.corrcoef(n[0::2], n[1::2])[0, 1]) < 5 * math.sqrt(2.0) * se


def test_normals_prefix_stable():
    a = rng.normals(9, 11)
    b = rng.normals(9, 12)
    assert np.array_equal(a, b[:11])


# ---------------------------------------------------------------- Cl(3,0)

def _basis(i):
    e = np.zeros(8)
    e[i] = 1.0
    return e


def test_blade_table_by_hand():
    e1, e2, e3, e12, e13, e23, e123 = (_basis(i) for i in range(1, 8))
    one = _basis(0)
    for e in (e1, e2, e3):
        assert np.array_equal(clifford.gp(e, e), one)  # e_i e_i = +1
    assert np.array_equal(clifford.gp(e1, e2), e12)
    assert np.array_equal(clifford.gp(e2, e1), -e12)
    assert np.array_equal(clifford.gp(e1, e3), e13)
    assert np.array_equal(clifford.gp(e3, e2), -e23)
    assert np.array_equal(clifford.gp(e12, e12), -one)
    assert np.array_equal(clifford.gp(e123, e123), -one)
    assert np.array_equal(clifford.gp(e12, e3), e123)
    assert np.array_equal(clifford.gp(e1, e23), e123)
    assert np.array_equal(clifford.gp(e2, e13), -e123)


def test_product_is_associative_and_distributive():
    g = np.random.default_rng(3)
    a, b, c = g.normal(size=(3, 50, 8))
    lhs = clifford.gp(clifford.gp(a, b), c)
    rhs = clifford.gp(a, clifford.gp(b, c))
    assert np.abs(lhs - rhs).max() < 1e-12
    assert np.abs(clifford.gp(a, b + c) - clifford.gp(a, b) - clifford.gp(a, c)).max() < 1e-12


def test_reverse_is_an_anti_automorphism():
    g = np.random.default_rng(4)
    a, b = g.normal(size=(2, 20, 8))
    lhs = clifford.reverse(clifford.gp(a, b))
    rhs = clifford.gp(clifford.reverse(b), clifford.reverse(a))
    assert np.abs(lhs - rhs).max() < 1e-12


def test_sandwich_closed_form_plane_rotation():
    # R = cos(t/2) + sin(t/2) e12 maps e1 -> cos t e1 - sin t e2 (derived by hand:
    # R e1 = c e1 - s e2, then (c e1 - s e2)(c - s e12) = (c^2 - s^2) e1 - 2cs e2).
    for t in (0.6, 1.0, -2.3):
        R = clifford.rotor(math.cos(t / 2), math.sin(t / 2), 0.0, 0.0)
        out = clifford.sandwich(R, [1.0, 0.0, 0.0])
        assert np.allclose(out[1:4], [math.cos(t), -math.sin(t), 0.0], atol=1e-15)
    R = clifford.rotor(math.cos(0.3), math.sin(0.3), 0.0, 0.0)
    assert np.allclose(clifford.sandwich(R, [1.0, 0.0, 0.0])[1:4], [0.82533561, -0.56464247, 0.0], atol=1e-8)
    # e3 is orthogonal to the e12 plane and stays put
    assert np.allclose(clifford.sandwich(R, [0.0, 0.0, 1.0])[1:4], [0.0, 0.0, 1.0], atol=1e-15)


def _sandwich_matrix(r):
    R = clifford.rotor(*r)
    return np.stack([clifford.sandwich(R, e)[1:4] for e in np.eye(3)], axis=1)


def test_sandwich_is_a_rotation_matching_the_quaternion_matrix():
    # textbook Hamilton quaternion rotation matrix of (w, x, y, z)
    def qmat(w, x, y, z):
        return np.array([[1 - 2 * (y * y + z * z), 2 * (x * y - w * z), 2 * (x * z + w * y)],
                         [2 * (x * y + w * z), 1 - 2 * (x * x + z * z), 2 * (y * z - w * x)],
                         [2 * (x * z - w * y), 2 * (y * z + w * x), 1 - 2 * (x * x + y * y)]])
    rot = params.rotors(30, 11)
    for s, b12, b13, b23 in rot:
        M = _sandwich_matrix((s, b12, b13, b23))
        assert np.abs(M @ M.T - np.eye(3)).max() < 1e-14
        assert abs(np.linalg.det(M) - 1.0) < 1e-14
        assert np.abs(M - qmat(s, -b23, b13, -b12)).max() < 1e-14


def test_sandwich_preserves_norms_and_grades_and_inverts():
    g = np.random.default_rng(5)
    rot = params.rotors(300, 12)
    R = clifford.rotor(rot[:, 0], rot[:, 1], rot[:, 2], rot[:, 3])
    v = g.normal(size=(rot.shape[0], 3))
    w = clifford.sandwich(R, v)
    assert np.abs(w[:, [0, 4, 5, 6, 7]]).max() < 1e-14
    assert np.abs(np.linalg.norm(w[:, 1:4], axis=1) - np.linalg.norm(v, axis=1)).max() < 1e-13
    back = clifford.unsandwich(R, w[:, 1:4])
    assert np.abs(back[:, 1:4] - v).max() < 1e-14
    # inner products are preserved too
    v2 = g.normal(size=v.shape)
    w2 = clifford.sandwich(R, v2)
    assert np.abs(np.sum(w[:, 1:4] * w2[:, 1:4], 1) - np.sum(v * v2, 1)).max() < 1e-13


def test_negative_control_wrong_product_order_is_not_the_sandwich():
    # "Non-Commutative Algebra Bug Fix": R~ (R v) is not the sandwich (R v) R~
    rot = params.rotors(30, 13)
    R = clifford.rotor(rot[:, 0], rot[:, 1], rot[:, 2], rot[:, 3])
    v = np.random.default_rng(6).normal(size=(rot.shape[0], 3))
    wrong = clifford.gp(clifford.reverse(R), clifford.gp(R, clifford.embed_vector(v)))
    right = clifford.sandwich(R, v)
    assert np.abs(wrong - right).max() > 0.1
    # the wrong form is just the identity on the vector part here, so the
    # inverse check used on the right form fails for it
    assert np.abs(clifford.unsandwich(R, wrong[:, 1:4])[:, 1:4] - v).max() > 0.1


# ---------------------------------------------------------------- parameters

def test_rotors_unit_and_group_count():
    for d, G in ((3, 1), (4, 2), (128, 43), (129, 43), (256, 86), (1536, 512), (4096, 1366)):
        r = params.rotors(d, 1)
        assert r.shape == (G, 4)
        assert np.abs(np.linalg.norm(r, axis=1) - 1).max() < 1e-15


def test_rotation_orthogonal_with_positive_r_diagonal():
    for d in (2, 3, 17, 128):
        Pi = params.rotation(d, 2)
        assert np.abs(Pi @ Pi.T - np.eye(d)).max() < 1e-13
        A = rng.normals(2, d * d).reshape(d, d)
        R = Pi.T @ A  # A = Pi R
        assert np.abs(np.tril(R, -1)).max() < 1e-12
        assert np.diag(R).min() > 0


def test_qjl_matrix_is_the_stream_row_major():
    T = params.qjl_matrix(4, 6, 3)
    assert np.array_equal(T.reshape(-1), rng.normals(3, 24))
