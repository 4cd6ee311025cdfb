"""The comparison rules of tests/parity.py on the CPU: a float32 restatement of the kernel's
arithmetic passes them, and a planted error fails them."""

import numpy as np
import pytest

from oracle import codebook, codes as ocodes, params, tq
from tests.parity import compare_sketch_signs, residual_sketch_slack


def _fp16(a):
    return np.asarray(a).astype(np.float16).astype(np.float64)


def _float32_prod_signs(x, Pi, T, c):
    """Signs of TurboQuant-prod as a float32 pipeline forms them (fp16 operands, float32 sums)."""
    x32, Pi32, T32 = x.astype(np.float32), Pi.astype(np.float32), T.astype(np.float32)
    nrm = np.sqrt(np.sum(x32 * x32, axis=1, dtype=np.float32))
    y = (x32 @ Pi32.T) * (np.float32(1) / nrm)[:, None]
    t = 0.5 * (c[:-1] + c[1:]).astype(np.float32)
    idx = np.searchsorted(t, y)
    r = (y - c.astype(np.float32)[idx]) * np.float32(256)
    rho = r.astype(np.float16).astype(np.float32)
    p = rho @ T32.T
    return ocodes.pack((p >= 0).astype(np.int64), 1), idx


@pytest.mark.parametrize("d", [128, 256])
def test_float32_pipeline_signs_pass(d):
    rng = np.random.default_rng(d)
    x = _fp16(rng.standard_normal((400, d)))
    Pi = _fp16(params.rotation(d, 2))
    T = _fp16(params.qjl_matrix(d, d, 3))
    c = codebook.lloyd_max(d, 2)[0].astype(np.float32).astype(np.float64)
    ref = tq.prod_quantize(x, Pi, T, c, 3)
    words, idx = _float32_prod_signs(x, Pi, T, c)
    bad_rows = np.any(idx != ref["codes"], axis=1)
    compare_sketch_signs(words, ref, x, Pi, T, c, skip_rows=bad_rows)
    # the bound is small against the spread of p: the rule accepts only signs near zero
    p, bound = residual_sketch_slack(ref, x, Pi, T, c)
    assert np.median(bound) < 1e-2 * np.median(np.abs(p))


def test_planted_sign_error_fails():
    d = 128
    rng = np.random.default_rng(7)
    x = _fp16(rng.standard_normal((64, d)))
    Pi = _fp16(params.rotation(d, 2))
    T = _fp16(params.qjl_matrix(d, d, 3))
    c = codebook.lloyd_max(d, 2)[0]
    ref = tq.prod_quantize(x, Pi, T, c, 3)
    p, bound = residual_sketch_slack(ref, x, Pi, T, c)
    s = ocodes.unpack(ref["signs_words"], d, 1)
    i, j = np.unravel_index(np.argmax(np.abs(p) - bound), p.shape)  # the sign farthest from its bound
    s[i, j] ^= 1
    with pytest.raises(AssertionError, match="beyond the rounding bound"):
        compare_sketch_signs(ocodes.pack(s, 1), ref, x, Pi, T, c, report=False)
    # many flips, each inside its bound, exceed the count limit
    x = _fp16(rng.standard_normal((2000, d)))
    ref = tq.prod_quantize(x, Pi, T, c, 3)
    p, bound = residual_sketch_slack(ref, x, Pi, T, c)
    inside = np.flatnonzero(np.abs(p).ravel() <= bound.ravel())
    assert inside.size > 8
    s = ocodes.unpack(ref["signs_words"], d, 1)
    s.ravel()[inside] ^= 1
    compare_sketch_signs(ocodes.pack(s, 1), ref, x, Pi, T, c, max_frac=1.0, report=False)
    with pytest.raises(AssertionError, match="signs differ"):
        compare_sketch_signs(ocodes.pack(s, 1), ref, x, Pi, T, c, max_frac=0.0, report=False)


def _fp16_scores(method, q, keys, p, bits):
    """Packed-code scores as the tensor-core kernel forms them: fp16 rotated query, fp16 centroids (and fp16
    T q' against the +-1 signs), float32 sums and epilogue."""
    from oracle import rq as orq
    from oracle.params import n_groups
    d = q.shape[1]
    c16 = np.asarray(p["centroids"]).astype(np.float16).astype(np.float32)
    out = []
    for h in range(q.shape[0]):
        if method == "rq":
            qp = orq.rotate(q[h:h + 1], p["rotors"])[0]
            idx = ocodes.unpack(keys["words"][0], 3 * n_groups(d), bits)
        else:
            qp = p["Pi"] @ q[h]
            idx = ocodes.unpack(keys["words"][0], d, bits if method == "tq_mse" else bits - 1)
        qp16 = qp.astype(np.float16).astype(np.float32)
        s = (c16[idx] @ qp16).astype(np.float32)
        if method == "tq_prod":
            T = np.asarray(p["T"])
            tq16 = (T.astype(np.float32) @ qp.astype(np.float32)).astype(np.float16).astype(np.float32)
            sg = (2 * ocodes.unpack(keys["signs_words"][0], T.shape[0], 1) - 1).astype(np.float32)
            s = s + np.float32(tq.QJL_SCALE_NUM / T.shape[0]) * keys["gammas"][0].astype(np.float32) * (sg @ tq16)
        out.append(keys["norms"][0].astype(np.float32) * s)
    return np.stack(out).astype(np.float64)


@pytest.mark.parametrize("method,bits", [("rq", 3), ("tq_mse", 3), ("tq_prod", 3), ("tq_prod", 2)])
def test_score_tolerance_accepts_fp16_restatement(method, bits):
    from oracle import rq as orq, score
    from tests.parity import compare_scores, score_tolerance
    d, n = 128, 3000
    rng = np.random.default_rng(5)
    c = codebook.lloyd_max(d, bits - 1 if method == "tq_prod" else bits)[0].astype(np.float32).astype(np.float64)
    p = {"centroids": c, "rotors": params.rotors(d, 1).astype(np.float32).astype(np.float64),
         "Pi": _fp16(params.rotation(d, 2)), "T": _fp16(params.qjl_matrix(d, d, 3))}
    k = rng.standard_normal((n, d)) * np.exp(0.5 * rng.standard_normal((n, 1)))
    if method == "rq":
        qq = orq.quantize(k, p["rotors"], c, bits)
    elif method == "tq_mse":
        qq = tq.mse_quantize(k, p["Pi"], c, bits)
    else:
        qq = tq.prod_quantize(k, p["Pi"], p["T"], c, bits)
    keys = {"words": qq["words"][None], "norms": qq["norms"].astype(np.float32).astype(np.float64)[None]}
    if method == "tq_prod":
        keys["signs_words"] = qq["signs_words"][None]
        keys["gammas"] = qq["gammas"].astype(np.float32).astype(np.float64)[None]
    q = _fp16(rng.standard_normal((8, d)))
    ref = score.direct(method, q, keys, p, bits)
    floor = score_tolerance(method, q, keys, p, bits)
    got = _fp16_scores(method, q, keys, p, bits)
    worst = compare_scores(got, ref, floor)
    assert worst < 1e-2  # the tensor-core bound of the scores, relative
    assert np.median(floor) < 1e-2 * np.median(np.abs(ref))
    # planted mistakes fail: a code moved to its neighbour, and (prod) one sign flipped
    w = qq["words"].copy()
    w[17, 0] ^= 1
    bad = dict(keys, words=w[None])
    with pytest.raises(AssertionError):
        compare_scores(score.direct(method, q, bad, p, bits), ref, floor, report=False)
    if method == "tq_prod":
        sw = qq["signs_words"].copy()
        sw[5, 1] ^= 1 << 7
        with pytest.raises(AssertionError):
            compare_scores(score.direct(method, q, dict(keys, signs_words=sw[None]), p, bits), ref, floor,
                           report=False)


def _float32_polar_words(x, Pi, books32):
    """PolarQuant code rows as a float32 pipeline forms them: y = Pi x in float32, level-1 sectors against
    tan(pi/8), 1, tan(3 pi/8), level >= 2 codes by comparing b cos t with a sin t, float32 radii."""
    F = np.float32
    y = (x.astype(F) @ Pi.astype(F).T).astype(F)
    t8, t38 = F(np.tan(np.pi / 8)), F(np.tan(3 * np.pi / 8))
    n = x.shape[0]
    words = np.zeros((n, 16), dtype=np.uint32)
    a, b = y[:, 0::2], y[:, 1::2]
    q = np.where(b >= 0, np.where((a > 0) | (b == 0), 0, 1), np.where(a < 0, 2, 3))
    xx = np.choose(q, [a, b, -a, -b]).astype(F)
    yy = np.choose(q, [b, -a, -b, a]).astype(F)
    k1 = 4 * q + (yy > (xx * t8).astype(F)) + (yy > xx) + (yy > (xx * t38).astype(F))
    r = np.sqrt((a * a + b * b).astype(F)).astype(F)
    codes = [k1]
    for lv in range(1, 4):
        c = books32[lv]
        t = (F(0.5) * (c[:-1] + c[1:])).astype(F)
        ct, st = np.cos(t).astype(F), np.sin(t).astype(F)
        ra, rb = r[:, 0::2], r[:, 1::2]
        h1 = (rb * ct[1]).astype(F) > (ra * st[1]).astype(F)
        hi = (rb * ct[2]).astype(F) > (ra * st[2]).astype(F)
        lo = (rb * ct[0]).astype(F) > (ra * st[0]).astype(F)
        codes.append(np.where(h1, 2 + hi, lo.astype(int)))
        r = np.sqrt((ra * ra + rb * rb).astype(F)).astype(F)
    words[:, 0:8] = ocodes.pack(codes[0], 4)
    words[:, 8:10] = ocodes.pack(codes[1], 2)
    words[:, 10:11] = ocodes.pack(codes[2], 2)
    words[:, 11:12] = ocodes.pack(codes[3], 2)
    h = r.astype(np.float16).view(np.uint16).astype(np.uint32)
    words[:, 12:16] = h[:, 0::2] | (h[:, 1::2] << 16)
    return words


def test_polar_rule_accepts_float32_restatement_and_rejects_planted_errors():
    from oracle import polar
    from tests.parity import compare_polar_codes, polar_angle_margins
    d = 128
    rng = np.random.default_rng(3)
    x = _fp16(rng.standard_normal((2000, d)) * np.exp(0.5 * rng.standard_normal((2000, 1))))
    x[10] = 0
    Pi = _fp16(params.rotation(d, 2))
    books32 = [polar.lloyd_max_angles(lv, b)[0].astype(np.float32) for lv, b in enumerate((4, 2, 2, 2), 1)]
    books = [b.astype(np.float64) for b in books32]
    ref = polar.quantize(x, Pi, books)
    margins = polar_angle_margins(x, Pi, ref)
    words = _float32_polar_words(x, Pi, books32)
    compare_polar_codes(words, ref, books, margins)
    assert np.median(margins[0]) < 1e-4  # the margins stay small for typical pairs
    # a level-2 code moved away from its boundary, and a radius moved by two fp16 steps, fail
    th = np.asarray(ref["angles"][1])
    t = 0.5 * (books[1][:-1] + books[1][1:])
    far = np.min(np.abs(th[..., None] - t), axis=-1) > 1e-2
    i, j = np.argwhere(far)[0]
    bad = words.copy()
    cd = ocodes.unpack(bad[:, 8:10], 32, 2)
    cd[i, j] = (cd[i, j] + 1) % 4
    bad[:, 8:10] = ocodes.pack(cd, 2)
    with pytest.raises(AssertionError):
        compare_polar_codes(bad, ref, books, margins)
    bad = words.copy()
    bad[5, 12] += 2
    with pytest.raises(AssertionError):
        compare_polar_codes(bad, ref, books, margins)
