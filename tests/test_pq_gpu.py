"""GPU parity of PolarQuant at d = 128 (pq_quantize_dequantize, pq_dequantize) against oracle/polar.py,
through the C ABI ("TurboQuant и PolarQuant: математика квантизации KV-кэша в LLM": "Полярное
преобразование", "Шаг 3: построение кодовых книг", "Степень сжатия").

Reconstructions are compared normwise with the oracle's reconstruction of the same codes: the rebuilt
y_hat enters the second tensor-core product rounded to the vector type (2^-11 relative for fp16,
2^-8 for bf16), so 2e-3 (fp16) and 1e-2 (bf16)."""

import functools

import numpy as np
import pytest
import torch

import kv_cache_vector_rq_b200 as kvrq
from kv_cache_vector_rq_b200 import synth
from oracle import params, polar
from tests.parity import compare_polar_codes, device_words, polar_angle_margins, random_words, to_f64, words_u32

pytestmark = pytest.mark.gpu

D = 128
XHAT_RTOL = {torch.float16: 2e-3, torch.bfloat16: 1e-2}


@functools.lru_cache(maxsize=None)
def _books32():
    return kvrq.pq_codebooks()


def _params(dt):
    c32 = _books32()
    books = [c32[:16], c32[16:20], c32[20:24], c32[24:28]]
    books64 = [b.astype(np.float64) for b in books]
    pi = torch.from_numpy(params.rotation(D, 2)).to(dt)
    return books64, pi.double().numpy(), pi.cuda(), torch.from_numpy(c32).cuda()


def _normwise(gpu, ref, rtol, skip=None):
    g, r = np.asarray(gpu, np.float64), np.asarray(ref, np.float64)
    keep = np.ones(len(g), bool) if skip is None else ~skip
    rn = np.linalg.norm(r[keep], axis=1)
    err = np.linalg.norm(g[keep] - r[keep], axis=1)
    ok = rn > 0
    assert np.all(err[ok] <= rtol * rn[ok]), "normwise relative error %g" % (err[ok] / rn[ok]).max()
    assert np.all(err[~ok] == 0)


def _check(x, rows=None):
    dt = x.dtype
    books64, pi64, pi_d, c_d = _params(dt)
    codes, xhat = kvrq.pq_quantize_dequantize(x, pi_d, c_d)
    torch.cuda.synchronize()
    kvrq.device_status()
    n = x.shape[0]
    rows = np.arange(n) if rows is None else rows
    idx = torch.as_tensor(rows, device="cuda")
    x64 = to_f64(x[idx])
    ref = polar.quantize(x64, pi64, books64)
    bad = compare_polar_codes(words_u32(codes[idx]), ref, books64, polar_angle_margins(x64, pi64, ref))
    xref = polar.dequantize(ref, pi64, books64)
    _normwise(to_f64(xhat[idx]), xref, XHAT_RTOL[dt], skip=bad)
    # dequantize-only of the fused launch's codes reproduces its x_hat bit for bit
    xd = kvrq.pq_dequantize(codes, D, pi_d, c_d, out_dtype=dt)
    torch.cuda.synchronize()
    assert torch.equal(xd.view(torch.int16), xhat.view(torch.int16))
    return codes, xhat, ref


@pytest.mark.parametrize("dt", [torch.float16, torch.bfloat16])
@pytest.mark.parametrize("n", [1, 100, 128, 129, 3000])
def test_roundtrip_matches_oracle(dt, n):
    _check(synth.lognormal(n, D, seed=n, dtype=dt).cuda())


def test_config2_full_size_sampled():
    x = synth.lognormal(65536, D, seed=0, dtype=torch.float16).cuda()
    rows = np.unique(np.concatenate([np.random.default_rng(3).choice(65536, 2048, replace=False), [0, 65535]]))
    _check(x, rows)


def test_unit_vector_quality():
    """Gaussian rows: unit-vector MSE and cosine of the GPU roundtrip near the oracle's (0.032, 0.984)."""
    x = synth.gaussian(4096, D, seed=11, dtype=torch.float16).cuda()
    _, xhat, _ = _check(x)
    xf, xh = to_f64(x), to_f64(xhat)
    nrm = np.linalg.norm(xf, axis=1, keepdims=True)
    mse = np.mean(np.sum((xf / nrm - xh / nrm) ** 2, axis=1))
    cos = np.mean(np.sum(xf * xh, axis=1) / (nrm[:, 0] * np.linalg.norm(xh, axis=1)))
    assert abs(mse - 0.032) < 0.004 and abs(cos - 0.984) < 0.003, (mse, cos)


def test_zero_rows():
    x = synth.lognormal(300, D, seed=5, dtype=torch.float16)
    x[[0, 7, 299]] = 0
    codes, xhat, _ = _check(x.cuda())
    w = words_u32(codes)[[0, 7, 299]]
    assert np.all(w == 0)  # every angle of a zero pair is 0 (code 0), every radius 0
    assert np.all(to_f64(xhat)[[0, 7, 299]] == 0)


@pytest.mark.parametrize("dt", [torch.float16, torch.bfloat16])
def test_dequantize_of_random_codes(dt):
    """Any code row with finite non-negative radii is a valid input: seeded random codes and LogNormal fp16
    radii, against the oracle's reconstruction."""
    books64, pi64, pi_d, c_d = _params(dt)
    g = np.random.default_rng(7)
    n = 1000
    w = np.zeros((n, 16), dtype=np.uint32)
    w[:, 0:8] = random_words(g, (n,), 64, 4)
    w[:, 8:10] = random_words(g, (n,), 32, 2)
    w[:, 10:11] = random_words(g, (n,), 16, 2)
    w[:, 11:12] = random_words(g, (n,), 8, 2)
    radii = np.exp(0.5 * g.standard_normal((n, 8))).astype(np.float16)
    w[:, 12:16] = radii.view(np.uint16).reshape(n, 4, 2).astype(np.uint32)[..., 0] | (
        radii.view(np.uint16).reshape(n, 4, 2).astype(np.uint32)[..., 1] << 16)
    xh = kvrq.pq_dequantize(device_words(w), D, pi_d, c_d, out_dtype=dt)
    torch.cuda.synchronize()
    from oracle import codes as ocodes
    q = {"codes": [ocodes.unpack(w[:, 0:8], 64, 4), ocodes.unpack(w[:, 8:10], 32, 2),
                   ocodes.unpack(w[:, 10:11], 16, 2), ocodes.unpack(w[:, 11:12], 8, 2)],
         "radii": radii.astype(np.float64)}
    _normwise(to_f64(xh), polar.dequantize(q, pi64, books64), XHAT_RTOL[dt])


def test_unsupported_shapes_are_rejected():
    books64, pi64, pi_d, c_d = _params(torch.float16)
    with pytest.raises(kvrq.KvrqError):
        kvrq.pq_quantize_dequantize(torch.zeros((4, 256), dtype=torch.float16, device="cuda"), pi_d, c_d)
    with pytest.raises(kvrq.KvrqError):
        kvrq.pq_quantize_dequantize(torch.zeros((4, D), dtype=torch.float32, device="cuda"), pi_d, c_d)


def test_axis_and_diagonal_pairs_with_identity_rotation():
    """Pi = I makes y = x exactly, so pairs can sit on the axes and the diagonals (boundaries of the level-1
    cells, and of the middle level-2 cell by the symmetry of its density): every quadrant's sign pattern,
    zeros of either sign, and equal radii. The angle of a boundary pair may take either neighbouring code; a
    zero pair takes code 0."""
    books64, _, _, c_d = _params(torch.float16)
    eye = torch.eye(D, dtype=torch.float16)
    g = np.random.default_rng(21)
    n = 512
    x = np.exp(0.5 * g.standard_normal((n, D))) * np.where(g.random((n, D)) < 0.5, -1.0, 1.0)
    pats = np.array([[1, 0], [0, 1], [-1, 0], [0, -1], [1, 1], [-1, 1], [-1, -1], [1, -1], [0, 0]], dtype=np.float64)
    for i in range(n):
        for p in range(D // 2):
            if g.random() < 0.6:
                x[i, 2 * p:2 * p + 2] = pats[g.integers(len(pats))] * x[i, 2 * p]
    x[5] = 0.0
    x[6, 0::2] = 2.0  # every pair (2, 1): equal radii at every level >= 2
    x[6, 1::2] = 1.0
    x[7, 0::2], x[7, 1::2] = -0.0, 3.0  # signed zeros against nonzero partners
    x[8, 0::2], x[8, 1::2] = 3.0, -0.0
    xt = torch.from_numpy(x).to(torch.float16)
    codes, xhat = kvrq.pq_quantize_dequantize(xt.cuda(), eye.cuda(), c_d)
    torch.cuda.synchronize()
    kvrq.device_status()
    x64 = xt.double().numpy()
    ref = polar.quantize(x64, np.eye(D), books64)
    w = words_u32(codes)
    bad = compare_polar_codes(w, ref, books64, polar_angle_margins(x64, np.eye(D), ref))
    assert np.all(w[5] == 0)
    _normwise(to_f64(xhat), polar.dequantize(ref, np.eye(D), books64), XHAT_RTOL[torch.float16], skip=bad)
    xd = kvrq.pq_dequantize(codes, D, eye.cuda(), c_d, out_dtype=torch.float16)
    torch.cuda.synchronize()
    assert torch.equal(xd.view(torch.int16), xhat.view(torch.int16))


@pytest.mark.parametrize("ld,off", [(17, 0), (20, 1)])
def test_strided_code_rows(ld, off):
    """Code rows with a stride that is not a multiple of four words, or not 16-byte aligned, take the
    word-by-word path: the same words as the contiguous layout, and the same x_hat from them."""
    books64, pi64, pi_d, c_d = _params(torch.float16)
    x = synth.lognormal(1000, D, seed=31, dtype=torch.float16).cuda()
    c0, x0 = kvrq.pq_quantize_dequantize(x, pi_d, c_d)
    buf = torch.full((1000, ld), -1, dtype=torch.int32, device="cuda")
    view = buf[:, off:off + 16]
    _, x1 = kvrq.pq_quantize_dequantize(x, pi_d, c_d, codes=view)
    torch.cuda.synchronize()
    assert torch.equal(view, c0) and torch.equal(x1.view(torch.int16), x0.view(torch.int16))
    rest = torch.cat([buf[:, :off], buf[:, off + 16:]], dim=1)
    assert torch.all(rest == -1)  # nothing outside the 16 words of a row is written
    xd = kvrq.pq_dequantize(view, D, pi_d, c_d, out_dtype=torch.float16)
    torch.cuda.synchronize()
    assert torch.equal(xd.view(torch.int16), x0.view(torch.int16))


def test_many_tiles_per_cta():
    """200,003 rows: five or six tiles per CTA through both tile buffers, ragged last tile."""
    x = synth.lognormal(200003, D, seed=13, dtype=torch.float16).cuda()
    rows = np.unique(np.concatenate([np.random.default_rng(4).choice(200003, 2048, replace=False), [0, 200002]]))
    _check(x, rows)
