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
    ref = tq.prod_quantize(x, Pi, T, c, 3, sketch_operand="f16")
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
    ref = tq.prod_quantize(x, Pi, T, c, 3, sketch_operand="f16")
    p, bound = residual_sketch_slack(ref, x, Pi, T, c)
    s = ocodes.unpack(ref["signs_words"], d, 1)
    i, j = np.unravel_index(np.argmax(np.abs(p) - bound), p.shape)  # the sign farthest from its bound
    s[i, j] ^= 1
    with pytest.raises(AssertionError, match="beyond the rounding bound"):
        compare_sketch_signs(ocodes.pack(s, 1), ref, x, Pi, T, c)
    # many flips, each inside its bound, exceed the count limit
    x = _fp16(rng.standard_normal((2000, d)))
    ref = tq.prod_quantize(x, Pi, T, c, 3, sketch_operand="f16")
    p, bound = residual_sketch_slack(ref, x, Pi, T, c)
    inside = np.flatnonzero(np.abs(p).ravel() <= bound.ravel())
    assert inside.size > 8
    s = ocodes.unpack(ref["signs_words"], d, 1)
    s.ravel()[inside] ^= 1
    compare_sketch_signs(ocodes.pack(s, 1), ref, x, Pi, T, c, max_frac=1.0)
    with pytest.raises(AssertionError, match="signs differ"):
        compare_sketch_signs(ocodes.pack(s, 1), ref, x, Pi, T, c, max_frac=0.0)
