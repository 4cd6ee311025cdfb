"""Pins for the oracle's quantizers, packing, QJL and scores (CPU only)."""

import itertools
import math
import os

import numpy as np
import pytest

from oracle import codebook, codes, params, rq, score, tq

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rows(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return [ln.split() for ln in f if ln.strip() and not ln.startswith("#")]


def _gauss(n, d, seed):
    return np.random.default_rng(seed).normal(size=(n, d))


# ---------------------------------------------------------------- codes

def test_nearest_tie_goes_to_lower_index():
    c = np.array([-1.0, 0.0, 1.0, 3.0])
    assert list(codes.nearest([-0.5, 0.5, 2.0, 5.0, -7.0, 0.49], c)) == [0, 1, 2, 3, 0, 1]


def test_pack_hand_example():
    # codes 1,2,3,4,5 at 3 bits, LSB first: bits 0 | 4 | 6,7 | 11 | 12,14
    w = codes.pack(np.array([[1, 2, 3, 4, 5]]), 3)
    assert w.shape == (1, 1) and int(w[0, 0]) == 1 + 16 + 64 + 128 + 2048 + 4096 + 16384
    # code 10 at 3 bits straddles words: bits 30, 31 | 32
    c = np.zeros((1, 11), dtype=np.int64)
    c[0, 10] = 0b111
    w = codes.pack(c, 3)
    assert w.shape == (1, 2) and int(w[0, 0]) == (3 << 30) and int(w[0, 1]) == 1


@pytest.mark.parametrize("n,bits", [(1, 1), (129, 3), (128, 2), (128, 4), (4098, 3), (37, 4)])
def test_pack_unpack_roundtrip_and_padding(n, bits):
    g = np.random.default_rng(n + bits)
    c = g.integers(0, 2 ** bits, size=(5, n))
    w = codes.pack(c, bits)
    assert w.shape == (5, codes.n_words(n, bits))
    assert np.array_equal(codes.unpack(w, n, bits), c)
    used = n * bits - 32 * (w.shape[1] - 1)
    if used < 32:
        assert np.all((w[:, -1].astype(np.int64) >> used) == 0)


# ---------------------------------------------------------------- RotorQuant

def test_rq_rotate_unrotate_identity_and_group_padding():
    d = 128
    u = _gauss(50, d, 1)
    rot = params.rotors(d, 1)
    y = rq.rotate(u, rot)
    assert y.shape == (50, 129)
    assert np.abs(np.linalg.norm(y, axis=1) - np.linalg.norm(u, axis=1)).max() < 1e-12
    assert np.abs(rq.unrotate(y, rot, d) - u).max() < 1e-13
    # group g only mixes coordinates 3g..3g+2
    u2 = u.copy()
    u2[:, 0] += 1.0
    y2 = rq.rotate(u2, rot)
    assert np.abs(y2[:, 3:] - y[:, 3:]).max() == 0.0


def test_rq_brute_force_tiny():
    # d = 3, b = 1: the per-coordinate nearest code is the nearest of all 8 codewords
    c, _, _ = codebook.lloyd_max(3, 1)
    rot = params.rotors(3, 4)
    x = _gauss(40, 3, 2)
    q = rq.quantize(x, rot, c, 1)
    words = codes.pack(q["codes"], 1)
    assert np.array_equal(words, q["words"])
    for i in range(x.shape[0]):
        best = min(itertools.product(range(2), repeat=3),
                   key=lambda k: np.sum((q["y"][i] - c[list(k)]) ** 2))
        assert list(q["codes"][i]) == list(best)
    xh = rq.dequantize(q["words"], q["norms"], rot, c, 1, 3)
    # reconstruction = norm * inverse rotation of the chosen codeword
    for i in range(3):
        ref = q["norms"][i] * rq.unrotate(c[q["codes"][i]][None], rot, 3)[0]
        assert np.allclose(xh[i], ref, atol=1e-15)


def test_rq_zero_vector_and_scale_invariance():
    c, _, _ = codebook.lloyd_max(128, 3)
    rot = params.rotors(128, 1)
    x = _gauss(8, 128, 3)
    x[3] = 0.0
    r = rq.roundtrip(x, rot, c, 3)
    assert r["norms"][3] == 0.0 and np.all(r["xhat"][3] == 0.0)
    assert np.all(r["codes"][3] == 3)  # y = 0 sits on the middle midpoint -> lower code
    r2 = rq.roundtrip(5.0 * x, rot, c, 3)
    assert np.array_equal(r2["codes"], r["codes"])
    assert np.abs(r2["xhat"] - 5.0 * r["xhat"]).max() < 1e-12


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_rq_and_tq_mse_quality_match_pages(bits):
    table = {int(r[0]): (float(r[1]), float(r[2]), float(r[3])) for r in _rows("mse_quality_table.txt")}
    tq_mse, rq_mse, cos = table[bits]
    d, n = 128, 20000
    x = _gauss(n, d, 10 + bits)
    u = x / np.linalg.norm(x, axis=1, keepdims=True)
    c, _, _ = codebook.lloyd_max(d, bits)
    D = d * codebook.distortion(c, d)
    # RotorQuant
    r = rq.roundtrip(u, params.rotors(d, 1), c, bits)
    err = np.sum((u - r["xhat"]) ** 2, axis=1)
    # the README prints 3 decimals: agree to within half a unit of the last one
    se = err.std() / math.sqrt(n)
    assert abs(err.mean() - rq_mse) <= 0.0005 + 4 * se
    assert abs(err.mean() / D - 1) < 0.02
    cosv = np.sum(u * r["xhat"], 1) / np.linalg.norm(r["xhat"], axis=1)
    assert abs(cosv.mean() - cos) < 0.0025
    # TurboQuant-mse
    Pi = params.rotation(d, 2)
    q = tq.mse_quantize(u, Pi, c, bits)
    xh = tq.mse_dequantize(q["words"], q["norms"], Pi, c, bits, d)
    err_t = np.sum((u - xh) ** 2, axis=1)
    assert abs(err_t.mean() - tq_mse) <= 0.0005 + 4 * err_t.std() / math.sqrt(n)
    assert abs(err_t.mean() / D - 1) < 0.02
    # Lloyd condition: E<u, x_tilde> = 1 - D (up to sampling error)
    assert abs(np.sum(u * xh, 1).mean() - (1 - D)) < 4 * np.sum(u * xh, 1).std() / math.sqrt(n)
    cos_t = np.sum(u * xh, 1) / np.linalg.norm(xh, axis=1)
    assert abs(cos_t.mean() - cos) < 0.0025


# ---------------------------------------------------------------- TurboQuant-prod / QJL

def test_prod_rotated_form_equals_pages_form_with_exact_pi():
    d, bits = 64, 3
    x = _gauss(30, d, 20)
    Pi = params.rotation(d, 2)
    T = params.qjl_matrix(d, d, 3)
    c, _, _ = codebook.lloyd_max(d, bits - 1)
    q = tq.prod_quantize(x, Pi, T, c, bits)
    xh = tq.prod_dequantize(q["words"], q["signs_words"], q["gammas"], q["norms"], Pi, T, c, bits, d)
    x_lit, r, qjl = tq.prod_quantize_literal(x, Pi, T, c)
    assert np.array_equal(q["signs"], qjl.astype(np.int64))
    assert np.abs(q["gammas"] - np.linalg.norm(r, axis=1)).max() < 1e-13
    assert np.abs(xh - q["norms"][:, None] * x_lit).max() < 1e-12


def test_qjl_unbiased_and_variance_bound():
    # "QJL 内积无偏估计（Theorem 2）": E_S <y, x_qjl> = <y, r>,
    # Var <= pi / (2m) ||r||^2 ||y||^2, over independent Gaussian S.
    d = m = 32
    g = np.random.default_rng(7)
    r = g.normal(size=d) * 0.1
    y = g.normal(size=d)
    K = 20000
    S = g.normal(size=(K, m, d))
    sg = np.where(np.einsum("kmd,d->km", S, r) >= 0, 1.0, -1.0)
    est = (tq.QJL_SCALE_NUM / m) * np.linalg.norm(r) * np.einsum("km,kmd,d->k", sg, S, y)
    bound_sd = math.sqrt(math.pi / (2 * m)) * np.linalg.norm(r) * np.linalg.norm(y)
    assert abs(est.mean() - y @ r) < 4 * bound_sd / math.sqrt(K)
    assert est.var() <= (math.pi / (2 * m)) * (np.linalg.norm(r) * np.linalg.norm(y)) ** 2 * 1.05
    # the scale matters: the pages' garbled sqrt((pi/2)/d) would be biased for m = d
    wrong = math.sqrt((math.pi / 2) / d) * np.linalg.norm(r) * np.einsum("km,kmd,d->k", sg, S, y)
    assert abs(wrong.mean() - y @ r) > 10 * bound_sd / math.sqrt(K)


def test_prod_is_unbiased_where_mse_is_shrunk():
    # MSE-only at 1 bit shrinks inner products by 1 - D_1 ~ 2/pi; adding the
    # QJL sketch removes the bias (averaging over independent T draws).
    d, bits = 128, 2
    g = np.random.default_rng(8)
    x = g.normal(size=(1, d))
    u = x / np.linalg.norm(x)
    yq = g.normal(size=d)
    c1, _, _ = codebook.lloyd_max(d, 1)
    D1 = d * codebook.distortion(c1, d)
    assert abs((1 - D1) - 2 / math.pi) < 0.003
    Pi = params.rotation(d, 2)
    q = tq.mse_quantize(u, Pi, c1, 1)
    x_mse = tq.mse_dequantize(q["words"], q["norms"], Pi, c1, 1, d)[0]
    r = u[0] - x_mse
    K = 4000
    est = np.empty(K)
    for k in range(K):
        T = g.normal(size=(d, d))
        s = np.where(T @ (Pi @ r) >= 0, 1.0, -1.0)
        est[k] = yq @ (x_mse + (tq.QJL_SCALE_NUM / d) * np.linalg.norm(r) * (Pi.T @ (T.T @ s)))
    sd = math.sqrt(math.pi / (2 * d)) * np.linalg.norm(r) * np.linalg.norm(yq)
    assert abs(est.mean() - yq @ u[0]) < 4 * sd / math.sqrt(K)
    # the MSE-only ratio over many unit vectors: E<u, x_mse> = 1 - D_1
    xs = g.normal(size=(20000, d))
    us = xs / np.linalg.norm(xs, axis=1, keepdims=True)
    qq = tq.mse_quantize(us, Pi, c1, 1)
    xm = tq.mse_dequantize(qq["words"], qq["norms"], Pi, c1, 1, d)
    assert abs(np.sum(us * xm, 1).mean() - (1 - D1)) < 0.002


def test_prod_distortion_bound():
    # D_prod <= sqrt(3) pi^2 ||y||^2 / d * 4^-b (Theorem 2 with the sqrt(3) pi / 2 reading)
    d, bits = 128, 3
    g = np.random.default_rng(9)
    c, _, _ = codebook.lloyd_max(d, bits - 1)
    Pi = params.rotation(d, 2)
    xs = g.normal(size=(400, d))
    us = xs / np.linalg.norm(xs, axis=1, keepdims=True)
    yq = g.normal(size=d)
    yq /= np.linalg.norm(yq)
    errs = []
    for k in range(10):
        T = g.normal(size=(d, d))
        q = tq.prod_quantize(us, Pi, T, c, bits)
        xh = tq.prod_dequantize(q["words"], q["signs_words"], q["gammas"], q["norms"], Pi, T, c, bits, d)
        errs.append((xh @ yq - us @ yq) ** 2)
    assert np.mean(errs) <= math.sqrt(3) * math.pi ** 2 / d * 4.0 ** -bits


def test_prod_zero_residual_and_sign_of_zero():
    d = 4
    Pi = np.eye(d)
    T = params.qjl_matrix(d, d, 3)
    c = np.array([-0.5, 0.5])
    x = np.array([[0.5, 0.5, -0.5, -0.5]])  # unit vector, every coordinate on a centroid
    q = tq.prod_quantize(x, Pi, T, c, 2)
    assert q["gammas"][0] == 0.0
    assert np.all(q["signs"] == 1)
    xh = tq.prod_dequantize(q["words"], q["signs_words"], q["gammas"], q["norms"], Pi, T, c, 2, d)
    assert np.array_equal(xh, x)


# ---------------------------------------------------------------- scores

@pytest.mark.parametrize("method,bits", [("rq", 3), ("tq_mse", 3), ("tq_prod", 3), ("rq", 2), ("tq_prod", 4)])
def test_score_direct_equals_reconstruct_with_gqa(method, bits):
    d, Hq, Hkv, n_tok = 128, 8, 2, 40
    g = np.random.default_rng(11)
    q = g.normal(size=(Hq, d))
    k = g.normal(size=(Hkv, n_tok, d)) * np.exp(g.normal(size=(Hkv, n_tok, 1)) * 0.5)
    b_store = bits - 1 if method == "tq_prod" else bits
    c, _, _ = codebook.lloyd_max(d, b_store)
    p = {"centroids": c, "rotors": params.rotors(d, 1), "Pi": params.rotation(d, 2), "T": params.qjl_matrix(d, d, 3)}
    keys = {"words": [], "norms": [], "signs_words": [], "gammas": []}
    for h in range(Hkv):
        if method == "rq":
            qq = rq.quantize(k[h], p["rotors"], c, bits)
        elif method == "tq_mse":
            qq = tq.mse_quantize(k[h], p["Pi"], c, bits)
        else:
            qq = tq.prod_quantize(k[h], p["Pi"], p["T"], c, bits)
            keys["signs_words"].append(qq["signs_words"])
            keys["gammas"].append(qq["gammas"])
        keys["words"].append(qq["words"])
        keys["norms"].append(qq["norms"])
    keys = {kk: np.stack(v) for kk, v in keys.items() if v}
    s1 = score.direct(method, q, keys, p, bits)
    s2 = score.reconstruct(method, q, keys, p, bits)
    assert s1.shape == (Hq, n_tok)
    assert np.abs(s1 - s2).max() < 1e-12 * np.abs(s2).max()
    # grouped-query mapping: heads 0..3 read KV head 0, heads 4..7 read KV head 1
    solo = score.direct(method, q[4:5], {kk: v[1:2] for kk, v in keys.items()}, p, bits)
    assert np.abs(solo[0] - s1[4]).max() == 0.0


def test_blog_worked_rotation_example():
    rows = {r[0]: [float(v) for v in r[1:]] for r in _rows("blog_rotation_example.txt")}
    x = np.array([rows["x"]])
    Pi = np.array(rows["Pi"]).reshape(2, 2)
    c = np.array([-0.8, -0.6, 0.6, 0.8])  # a codebook holding the exact values
    q = tq.mse_quantize(x, Pi, c, 2)
    assert q["norms"][0] == rows["norm"][0]
    assert np.allclose(q["y"][0], rows["y"], atol=1e-15)
    assert list(q["codes"][0]) == [0, 2]
    xh = tq.mse_dequantize(q["words"], q["norms"], Pi, c, 2, 2)
    assert np.allclose(xh[0], rows["x"], atol=1e-14)
