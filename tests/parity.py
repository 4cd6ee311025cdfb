"""Comparison rules between the CUDA path and the float64 oracle.

Codes: bit-exact, except at coordinates whose oracle decision value lies within
MARGIN (1e-5, unit-sphere scale) of a decision boundary; there either adjacent
code is accepted and the case is counted. Float outputs: within one unit in
the last place of the output dtype plus a float32-arithmetic allowance, on
rows whose codes all agree (normwise relative error is also bounded by
1e-3 plus the output dtype's unit roundoff).
"""

import numpy as np
import torch

from oracle import codes as ocodes

MARGIN = 1e-5

UNIT_ROUNDOFF = {torch.float32: 2.0 ** -24, torch.float16: 2.0 ** -11, torch.bfloat16: 2.0 ** -8}


def to_f64(t):
    return t.detach().to("cpu").to(torch.float64).numpy()


def words_u32(t):
    """int32 device/host tensor of packed words -> uint32 numpy."""
    return t.detach().to("cpu").numpy().astype(np.int64).astype(np.uint32)


def device_words(words, device="cuda"):
    """An oracle's uint32 code words uploaded as an int32 device tensor (same bits): the oracle's own
    codes become the kernel's input, so that no oracle input ever comes from the CUDA path."""
    a = np.ascontiguousarray(np.asarray(words, dtype=np.uint32))
    return torch.from_numpy(a.view(np.int32)).to(device)


def oracle_prod_inputs(ref, device="cuda"):
    """The oracle's TurboQuant-prod result `ref` as device inputs of the library's dequantize or score
    (codes, signs, gammas, norms; gammas and norms rounded to fp32 as the library stores them) and the
    float64 values of those rounded gammas and norms, for the oracle's side of the comparison."""
    g32 = np.asarray(ref["gammas"], dtype=np.float32)
    n32 = np.asarray(ref["norms"], dtype=np.float32)
    dev = (device_words(ref["words"], device), device_words(ref["signs_words"], device),
           torch.from_numpy(g32).to(device), torch.from_numpy(n32).to(device))
    return dev, g32.astype(np.float64), n32.astype(np.float64)


def attention_tolerance(ref, vmax, rel=1e-3):
    """Allowed |error| of decode-attention outputs ref [rows, d]: rel x the largest |output| of the row
    (the fp32 path's relative bound) plus 1e-5 x max|v_hat| (the rounding of a weighted sum of thousands
    of fp32 terms, about sqrt(T) 2^-24 max|v_hat|)."""
    return rel * np.abs(ref).max(axis=1, keepdims=True) + 1e-5 * vmax


def random_words(g, shape, n_codes, bits):
    """Seeded uniformly random packed code rows [*shape, W] (unused high bits of the last word zero): any bit
    pattern is a valid row of codes, so these are inputs that no implementation produced."""
    W = -(-n_codes * bits // 32)
    w = g.integers(0, 1 << 32, size=tuple(shape) + (W,), dtype=np.uint64).astype(np.uint32)
    spare = W * 32 - n_codes * bits
    if spare:
        w[..., -1] &= np.uint32((1 << (32 - spare)) - 1)
    return w


def ulp(values, dtype):
    """Spacing of `dtype` at |values| (float64 array)."""
    a = np.abs(values)
    if dtype == torch.float32:
        return np.spacing(a.astype(np.float32)).astype(np.float64)
    if dtype == torch.float16:
        return np.spacing(a.astype(np.float16)).astype(np.float64)
    # bfloat16: 8 significant bits, smallest normal 2^-126
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -126)))
    return 2.0 ** (e - 7)


def near_boundary(y, centroids, margin=MARGIN):
    """Boolean mask: the decision value y is within `margin` of a midpoint of the codebook."""
    c = np.asarray(centroids, dtype=np.float64)
    t = 0.5 * (c[:-1] + c[1:])
    if t.size == 0:
        return np.zeros(np.shape(y), dtype=bool)
    return np.min(np.abs(np.asarray(y)[..., None] - t), axis=-1) < margin


def compare_codes(gpu_words, oracle_q, n_codes, bits, centroids, decision=None, margin=MARGIN):
    """Checks GPU packed words against the oracle's quantization dict.

    Returns (n_boundary_mismatches, rows_with_any_mismatch mask). Raises
    AssertionError on any mismatch outside the margin, on a mismatch that is
    not to an adjacent code, or on nonzero padding bits."""
    gw = np.asarray(gpu_words, dtype=np.uint32)
    W = ocodes.n_words(n_codes, bits)
    assert gw.shape[1] >= W
    gw = gw[:, :W]
    used = n_codes * bits - 32 * (W - 1)
    if used < 32:
        assert np.all((gw[:, -1].astype(np.int64) >> used) == 0), "nonzero padding bits"
    g_codes = ocodes.unpack(gw, n_codes, bits)
    o_codes = oracle_q["codes"]
    y = oracle_q["y"] if decision is None else decision
    diff = g_codes != o_codes
    if diff.any():
        nb = near_boundary(y, centroids, margin)
        bad = diff & ~nb
        assert not bad.any(), "codes differ away from a decision boundary at %s (gpu %s, oracle %s, y %s)" % (
            np.argwhere(bad)[:5].tolist(), g_codes[bad][:5], o_codes[bad][:5], np.asarray(y)[bad][:5])
        assert np.all(np.abs(g_codes[diff] - o_codes[diff]) == 1), "boundary mismatch to a non-adjacent code"
    record("code boundary ties", int(diff.sum()), int(g_codes.size))
    return int(diff.sum()), diff.any(axis=1)


def compare_floats(gpu, ref, out_dtype, row_scale, skip_rows=None, arith_rtol=2e-6, name="x_hat"):
    """Elementwise |gpu - ref| <= ulp(ref) + arith_rtol * row_scale on rows not skipped,
    and normwise relative error <= 1e-3 + unit roundoff."""
    g = np.asarray(gpu, dtype=np.float64)
    r = np.asarray(ref, dtype=np.float64)
    keep = np.ones(g.shape[0], dtype=bool) if skip_rows is None else ~np.asarray(skip_rows)
    g, r = g[keep], r[keep]
    sc = np.asarray(row_scale, dtype=np.float64)[keep][:, None]
    tol = ulp(r, out_dtype) + arith_rtol * sc
    err = np.abs(g - r)
    assert np.all(err <= tol), "%s: max excess %g at %s" % (name, float(np.max(err - tol)),
                                                            np.unravel_index(np.argmax(err - tol), err.shape))
    rn = np.linalg.norm(r, axis=1)
    ok = rn > 0
    rel = np.linalg.norm(g - r, axis=1)[ok] / rn[ok]
    if rel.size:
        assert rel.max() <= 1e-3 + UNIT_ROUNDOFF[out_dtype], "%s: normwise relative error %g" % (name, rel.max())
    return int(keep.sum())


# Probabilistic rounding-error model of the float32 sums on the CUDA path
# (|error| <= LAMBDA * sqrt(n) * 2^-24 * sum |terms|, Higham & Mary 2019).
LAMBDA = 4.0


def residual_sketch_slack(ref, x64, Pi64, T64, centroids):
    """(p, bound): p = T r_rot in float64 (the oracle's decision values, ref["p"]) and a bound on |p| within
    which a CUDA path that projects fp16(2^8 r) with float32 arithmetic may take the other sign.

    The kernel forms y = Pi x with float32 sums of exact fp16 products, scales by 1/||x|| and subtracts the
    centroid, so each residual coordinate may differ from the float64 one by
    eps = LAMBDA sqrt(d) 2^-24 sum_k |Pi_ik u_k| + 2^-21 |y| + 2^-22 |c| (sums, then the norm, its
    reciprocal, the fma and the centroid chain). The tensor-core operand is then 2^8 r rounded to fp16;
    rounding is monotone, so it lies between fp16(2^8 (r - eps)) and fp16(2^8 (r + eps)), and the operand
    differs from 2^8 r by at most the larger distance to those two ends (this is where the fp16 step of the
    operand, at most 2^-11 relative per coordinate, enters). p_j then moves by at most sum_k |T_jk| times
    that distance, and the sketch's own float32 sums add LAMBDA sqrt(d) 2^-24 sum_k |T_jk 2^8 r_k|."""
    x64 = np.asarray(x64, dtype=np.float64)
    Pi64 = np.asarray(Pi64, dtype=np.float64)
    T64 = np.asarray(T64, dtype=np.float64)
    d = x64.shape[1]
    nrm = np.linalg.norm(x64, axis=1, keepdims=True)
    u = x64 / np.where(nrm > 0, nrm, 1.0)
    y = np.asarray(ref["y"], dtype=np.float64)
    c_hat = np.asarray(centroids, dtype=np.float64)[ref["codes"]]
    s = 256.0 * (y - c_hat)
    g = LAMBDA * np.sqrt(d) * 2.0 ** -24
    eps = g * (np.abs(u) @ np.abs(Pi64).T) + 2.0 ** -21 * np.abs(y) + 2.0 ** -22 * np.abs(c_hat)
    lo = (s - 256.0 * eps).astype(np.float16).astype(np.float64)
    hi = (s + 256.0 * eps).astype(np.float16).astype(np.float64)
    d_op = np.maximum(np.abs(hi - s), np.abs(lo - s))  # |operand - 2^8 r|, worst case
    aT = np.abs(T64).T
    p = np.asarray(ref["p"], dtype=np.float64)
    bound = (d_op @ aT + g * (np.abs(np.maximum(np.abs(lo), np.abs(hi))) @ aT)) / 256.0
    return p, bound


def compare_sketch_signs(gpu_sign_words, ref, x64, Pi64, T64, centroids, skip_rows=None, max_frac=2e-4,
                         report=True):
    """QJL signs of TurboQuant-prod against the plain definition sign(T r_rot) of the oracle: equal except
    where |T r_rot| is within the arithmetic's bound (residual_sketch_slack), and differing in at most
    max_frac of the signs compared (at least 8). Records and returns the number of differing signs.

    Expected rate: the fp16 operand's rounding errors are independent and uniform within half a unit in
    the last place, so p_j moves by about N(0, (0.21 2^-10 ||2^8 r||)^2) against p_j ~ N(0, ||2^8 r||^2);
    a sign flips with probability E|dp| phi(0) / ||2^8 r|| ~ 6.4e-5. max_frac = 2e-4 keeps a sample of
    10^5 signs about 5 standard deviations of the count away from a false failure."""
    T64 = np.asarray(T64, dtype=np.float64)
    m = T64.shape[0]
    gs = ocodes.unpack(np.asarray(gpu_sign_words, dtype=np.uint32), m, 1)
    os_ = ocodes.unpack(ref["signs_words"], m, 1)
    keep = np.ones(gs.shape[0], bool) if skip_rows is None else ~np.asarray(skip_rows)
    diff = (gs != os_) & keep[:, None]
    if diff.any():
        p, bound = residual_sketch_slack(ref, x64, Pi64, T64, centroids)
        far = diff & (np.abs(p) > bound)
        assert not far.any(), "sign differs beyond the rounding bound at %s (p %s, bound %s)" % (
            np.argwhere(far)[:5].tolist(), p[far][:5], bound[far][:5])
    n = int(diff.sum())
    total = int(keep.sum()) * m
    if report:
        record("qjl sign flips", n, total)
    assert n <= max(8, max_frac * total), "%d of %d signs differ" % (n, total)
    return n


# ---------------------------------------------------------------- scores

SCORE_RTOL = 1e-3
SCORE_SIGMAS = 6.0  # floor multiple of the fp16 roundings' spread (each at most 2^-11 relative)
SCORE_F32_REL = 2.0 ** -14  # float32 arithmetic: rotation, T q', tensor-core accumulation, epilogue


def score_tolerance(method, q, keys, params, bits):
    """Allowed |error| [Hq, T] of packed-code scores against oracle.score.direct: SCORE_RTOL |score| plus
    an absolute floor derived from the kernel's operands.

    The kernel multiplies fp16(q') by fp16(c_hat) (and, for TurboQuant-prod, fp16(T q') by the +-1 signs)
    with float32 accumulation, where q' is the rotated query. Per key, with n = ||k||, kappa = sqrt(pi/2)/m
    and gamma the residual norm, the floor is
      n |sum_i q'_i (fp16(c)_i - c_i)|      the centroid rounding, exact (one table of 2^b values)
    + n 6 2^-11 ||q' o fp16(c)||_2          the query rounding: independent, each at most 2^-11 relative
    + n kappa gamma 6 2^-11 ||T q'||_2      the rounding of T q'
    + n 2^-14 (sum |q'_i c_i| + kappa gamma sum_j |(T q')_j|)   float32 sums (14 significant bits kept
                                                               through the tensor-core accumulation).
    Six times the bound of each independent rounding is about 7 standard deviations of their sum."""
    from oracle import codes as oc, rq as orq, tq as otq
    from oracle.params import n_groups
    q = np.asarray(q, dtype=np.float64)
    Hq, d = q.shape
    words = np.asarray(keys["words"])
    Hkv = words.shape[0]
    c = np.asarray(params["centroids"], dtype=np.float64)
    c16 = c.astype(np.float16).astype(np.float64)
    u = 2.0 ** -11
    out = np.zeros((Hq, words.shape[1]))
    for h in range(Hq):
        kv = h // (Hq // Hkv)
        norms = np.asarray(keys["norms"], dtype=np.float64)[kv]
        if method == "rq":
            qp = orq.rotate(q[h:h + 1], params["rotors"])[0]
            idx = oc.unpack(words[kv], 3 * n_groups(d), bits)
        else:
            qp = np.asarray(params["Pi"], dtype=np.float64) @ q[h]
            idx = oc.unpack(words[kv], d, bits if method == "tq_mse" else bits - 1)
        a16 = c16[idx] * qp
        f = np.abs(a16.sum(axis=1) - (c[idx] * qp).sum(axis=1))
        f += SCORE_SIGMAS * u * np.sqrt(np.sum(a16 * a16, axis=1))
        f += SCORE_F32_REL * np.sum(np.abs(c[idx] * qp), axis=1)
        if method == "tq_prod":
            T = np.asarray(params["T"], dtype=np.float64)
            tq_ = T @ qp
            kg = (otq.QJL_SCALE_NUM / T.shape[0]) * np.asarray(keys["gammas"], dtype=np.float64)[kv]
            f += kg * (SCORE_SIGMAS * u * np.linalg.norm(tq_) + SCORE_F32_REL * np.sum(np.abs(tq_)))
        out[h] = norms * f
    return out


def compare_scores(got, ref, floor, rtol=SCORE_RTOL, name="scores", report=True):
    """|got - ref| <= rtol |ref| + floor elementwise; records the worst relative error over the scores of
    at least median magnitude (a score near zero has no relative accuracy from rounded operands), and the
    largest error as a fraction of its tolerance. Returns that worst relative error."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    tol = rtol * np.abs(ref) + floor
    err = np.abs(got - ref)
    big = (np.abs(ref) >= np.median(np.abs(ref))) & (ref != 0)
    worst_rel = float(np.max(err[big] / np.abs(ref[big]))) if big.any() else 0.0
    if report:
        record("scores worst rel err (|s| >= median)", worst_rel, int(big.sum()))
        record("scores max err / tol", float(np.max(err / tol)) if err.size else 0.0, int(err.size))
    assert np.all(err <= tol), "%s: max excess %g at %s (err/tol %g)" % (
        name, float(np.max(err - tol)), np.unravel_index(np.argmax(err - tol), err.shape), float(np.max(err / tol)))
    return worst_rel


# ---------------------------------------------------------------- reporting

REPORT = []


def record(kind, value, total):
    """Keeps a count (or worst value) of one comparison for the session summary printed by conftest."""
    import os
    test = os.environ.get("PYTEST_CURRENT_TEST", "?").split(" ")[0]
    REPORT.append((test, kind, value, total))


# ---------------------------------------------------------------- PolarQuant

def polar_angle_margins(x64, Pi64, ref):
    """Per level, a margin (radians) per angle within which the CUDA path may take the neighbouring code.

    The kernel forms y = Pi x with float32 sums of exact 16-bit products: |dy_i| <= e_i = LAMBDA sqrt(d) 2^-24
    sum_k |Pi_ik x_k|. A level-1 angle atan2(b, a) of a pair of radius r moves by at most (e_a + e_b) / r; a
    float32 radius carries the errors of its pair plus two roundings (2^-22 r), and a level-l angle of radii
    (r_a, r_b) moves by (dr_a + dr_b) / r. The decision itself (float32 products of the coordinates or
    squared radii with float32 tangents of the boundaries) adds 2^-21. Margin = max(1e-5, 2 x that bound)."""
    x64 = np.asarray(x64, dtype=np.float64)
    Pi64 = np.asarray(Pi64, dtype=np.float64)
    d = x64.shape[1]
    e = LAMBDA * np.sqrt(d) * 2.0 ** -24 * (np.abs(x64) @ np.abs(Pi64).T)
    y = x64 @ Pi64.T
    r = y
    dr = e
    out = []
    for level in range(len(ref["angles"])):
        a, b = r[:, 0::2], r[:, 1::2]
        da, db = dr[:, 0::2], dr[:, 1::2]
        rad = np.sqrt(a * a + b * b)
        with np.errstate(divide="ignore", invalid="ignore"):
            dth = np.where(rad > 0, (da + db) / rad, np.inf) + 2.0 ** -21
        out.append(np.maximum(1e-5, 2.0 * dth))
        dr = da + db + 2.0 ** -22 * rad
        r = rad
    return out


def compare_polar_codes(gpu_words, ref, books, margins):
    """GPU PolarQuant code rows [N, 16] against the oracle's quantization `ref`: every level's codes equal
    except where the oracle's angle is within its margin of a boundary (then the neighbouring code, modulo
    16 at level 1 whose boundaries include 0 = 2 pi), and the 16-bit radii equal or one fp16 step apart.
    Records the mismatches; returns the mask of rows with any."""
    gw = np.asarray(gpu_words, dtype=np.uint32)
    level_words = [(0, 8, 4), (8, 10, 2), (10, 11, 2), (11, 12, 2)]
    bad_rows = np.zeros(gw.shape[0], dtype=bool)
    total = 0
    for lv, (w0, w1, bits) in enumerate(level_words):
        n_codes = 64 >> lv
        g = ocodes.unpack(gw[:, w0:w1], n_codes, bits)
        o = np.asarray(ref["codes"][lv])
        diff = g != o
        if diff.any():
            c = np.asarray(books[lv], dtype=np.float64)
            t = 0.5 * (c[:-1] + c[1:])
            if lv == 0:
                t = np.concatenate([[0.0, 2.0 * np.pi], t])
            th = np.asarray(ref["angles"][lv])
            dist = np.min(np.abs(th[..., None] - t), axis=-1)
            far = diff & ~(dist < margins[lv])
            assert not far.any(), "level %d codes differ away from a boundary at %s (gpu %s, oracle %s)" % (
                lv + 1, np.argwhere(far)[:5].tolist(), g[far][:5], o[far][:5])
            step = np.abs(g[diff] - o[diff])
            if lv == 0:
                step = np.minimum(step, 16 - step)
            assert np.all(step == 1), "level %d: boundary mismatch to a non-adjacent code" % (lv + 1)
            bad_rows |= diff.any(axis=1)
        total += int(diff.sum())
    assert np.all((gw[:, 11] >> 16) == 0), "nonzero padding bits"
    rad = gw[:, 12:16].view(np.uint16).astype(np.int64)
    orad = np.asarray(ref["radii"]).astype(np.float16).view(np.uint16).astype(np.int64)
    assert np.all(np.abs(rad - orad) <= 1), "fp16 radii differ by more than one step"
    record("polar code boundary ties", total, int(gw.shape[0]) * 120)
    return bad_rows
