"""GPU parity of the tiled TurboQuant path (any d that is a multiple of 128, and
fp32 vectors) against the float64 oracle, through the C ABI."""

import functools

import numpy as np
import pytest
import torch

import kv_cache_vector_rq_b200 as kvrq
from kv_cache_vector_rq_b200 import synth
from oracle import codebook, codes as ocodes, params, tq
from tests.parity import compare_codes, compare_sketch_signs, oracle_prod_inputs, to_f64, words_u32

pytestmark = pytest.mark.gpu

# Normwise relative tolerance of reconstructions: the second product takes the
# centroids (or the QJL-corrected centroids) rounded to its operand type
# (fp16 2^-11, bf16 2^-8; fp32 vectors use an exact fp16 hi + lo split), plus
# the output's own rounding.
XHAT_RTOL = {torch.float32: 1e-5, torch.float16: 2e-3, torch.bfloat16: 1e-2}
SIGN_MARGIN = 1e-5  # decision cosine below which a sign may differ


@functools.lru_cache(maxsize=None)
def _pi64(d):
    return params.rotation(d, 2)


@functools.lru_cache(maxsize=None)
def _t64(d):
    return params.qjl_matrix(d, d, 3)


@functools.lru_cache(maxsize=None)
def _codebook(d, bits):
    return codebook.lloyd_max(d, bits)[0].astype(np.float32)


def _params(d, bits_store, dt):
    """Device parameters in the operand types, and the same rounded values as float64 for the oracle."""
    pdt = torch.float16 if dt == torch.float32 else dt
    pi_d = torch.from_numpy(_pi64(d)).to(pdt).cuda()
    T_d = torch.from_numpy(_t64(d)).to(torch.float16).cuda()
    c = _codebook(d, bits_store)
    return to_f64(pi_d), c.astype(np.float64), to_f64(T_d), pi_d, torch.from_numpy(c).cuda(), T_d


def _rows_close(gpu, ref, rtol, skip=None):
    g = np.asarray(gpu, dtype=np.float64)
    r = np.asarray(ref, dtype=np.float64)
    keep = np.ones(len(g), bool) if skip is None else ~np.asarray(skip)
    rn = np.linalg.norm(r[keep], axis=1)
    err = np.linalg.norm(g[keep] - r[keep], axis=1)
    ok = rn > 0
    assert np.all(err[ok] <= rtol * rn[ok]), "normwise relative error %g" % (err[ok] / rn[ok]).max()
    assert np.all(err[~ok] == 0)


def _input(n, d, dt, seed):
    if dt == torch.float32:
        return synth.gaussian(n, d, seed=seed, dtype=dt).cuda()
    return synth.lognormal(n, d, seed=seed, dtype=dt, outliers=()).cuda()


@pytest.mark.parametrize("d,dt,bits,n", [
    (256, torch.float16, 1, 300), (256, torch.float16, 2, 1000), (256, torch.bfloat16, 3, 777),
    (256, torch.float16, 4, 129), (384, torch.bfloat16, 2, 260), (384, torch.float16, 3, 1),
    (1536, torch.float16, 3, 300), (1536, torch.bfloat16, 4, 200), (4096, torch.float16, 2, 150),
    (128, torch.float32, 3, 1024), (256, torch.float32, 2, 333), (1536, torch.float32, 4, 130),
])
def test_mse_roundtrip_tiled(d, dt, bits, n):
    pi64, c64, _, pi_d, c_d, _ = _params(d, bits, dt)
    x = _input(n, d, dt, seed=d + bits + n)
    codes, norms, xhat = kvrq.tq_quantize_dequantize_mse(x, pi_d, c_d, bits)
    torch.cuda.synchronize()
    kvrq.device_status()
    ref = tq.mse_quantize(to_f64(x), pi64, c64, bits)
    nb, bad = compare_codes(words_u32(codes), ref, d, bits, c64)
    assert np.allclose(to_f64(norms), ref["norms"], rtol=1e-5)
    xref = tq.mse_dequantize(ref["words"], ref["norms"], pi64, c64, bits, d)
    _rows_close(to_f64(xhat), xref, XHAT_RTOL[dt], skip=bad)
    # quantize alone and dequantize of the codes give the same bits as the two-launch roundtrip
    c2, n2 = kvrq.tq_quantize_mse(x, pi_d, c_d, bits)
    assert torch.equal(c2, codes) and torch.equal(n2, norms)
    xd = kvrq.tq_dequantize(codes, norms, d, pi_d, c_d, bits, out_dtype=dt)
    assert torch.equal(xd, xhat)


def test_config1_fp32_tq_mse_quality():
    """1,024 N(0,1) fp32 vectors at d = 128, 3-bit TurboQuant-mse with a QR-derived Pi: the GPU's
    reconstruction has the oracle's MSE and cosine (per unit vector)."""
    d, bits, dt = 128, 3, torch.float32
    pi64, c64, _, pi_d, c_d, _ = _params(d, bits, dt)
    x = synth.gaussian(1024, d, seed=0, dtype=dt).cuda()
    codes, norms, xhat = kvrq.tq_quantize_dequantize_mse(x, pi_d, c_d, bits)
    torch.cuda.synchronize()
    x64 = to_f64(x)
    ref = tq.mse_quantize(x64, pi64, c64, bits)
    nb, bad = compare_codes(words_u32(codes), ref, d, bits, c64)
    xref = tq.mse_dequantize(ref["words"], ref["norms"], pi64, c64, bits, d)
    g = to_f64(xhat)
    nrm = np.linalg.norm(x64, axis=1)
    mse_gpu = np.mean(np.sum((g - x64) ** 2, axis=1) / nrm ** 2)
    mse_ref = np.mean(np.sum((xref - x64) ** 2, axis=1) / nrm ** 2)
    cos_gpu = np.mean(np.sum(g * x64, axis=1) / (np.linalg.norm(g, axis=1) * nrm))
    cos_ref = np.mean(np.sum(xref * x64, axis=1) / (np.linalg.norm(xref, axis=1) * nrm))
    assert abs(mse_gpu - mse_ref) <= 1e-4 * mse_ref
    assert abs(cos_gpu - cos_ref) <= 1e-6
    assert 0.025 < mse_ref < 0.045  # about 0.034 at 3 bits


@pytest.mark.parametrize("d,dt,bits,n,ws_rows", [
    (256, torch.float16, 3, 700, 256), (256, torch.bfloat16, 2, 300, None), (384, torch.float16, 4, 200, 128),
    (1536, torch.float16, 3, 260, 128), (1536, torch.bfloat16, 3, 130, None), (4096, torch.bfloat16, 2, 140, None),
    (128, torch.float32, 3, 500, 256), (256, torch.float32, 4, 200, None),
])
def test_prod_quantize_and_dequantize_tiled(d, dt, bits, n, ws_rows):
    pi64, c64, T64, pi_d, c_d, T_d = _params(d, bits - 1, dt)
    x = _input(n, d, dt, seed=n + d)
    ws = None
    if ws_rows is not None:  # a workspace smaller than n rows: several row blocks, a ragged last one
        ws = torch.empty((kvrq.tq_workspace_bytes(ws_rows, d),), dtype=torch.uint8, device="cuda")
    codes, signs, gammas, norms = kvrq.tq_quantize_prod(x, pi_d, T_d, c_d, bits, workspace=ws)
    torch.cuda.synchronize()
    kvrq.device_status()
    ref = tq.prod_quantize(to_f64(x), pi64, T64, c64, bits)
    nb, bad = compare_codes(words_u32(codes), ref, d, bits - 1, c64)
    assert np.allclose(to_f64(norms), ref["norms"], rtol=1e-5)
    g = to_f64(gammas)
    assert np.allclose(g[~bad], ref["gammas"][~bad], rtol=1e-4, atol=1e-7)
    compare_sketch_signs(words_u32(signs), ref, to_f64(x), pi64, T64, c64, skip_rows=bad)
    if ws_rows is not None:  # the row blocking does not change any bit
        c1, s1, g1, n1 = kvrq.tq_quantize_prod(x, pi_d, T_d, c_d, bits)
        assert torch.equal(c1, codes) and torch.equal(s1, signs) and torch.equal(g1, gammas)
        assert torch.equal(n1, norms)
    # dequantize the oracle's codes on the GPU, against the oracle's reconstruction of the same codes
    (oc, osg, og, on), g64, n64 = oracle_prod_inputs(ref)
    xh = kvrq.tq_dequantize(oc, on, d, pi_d, c_d, bits, signs=osg, gammas=og, T=T_d, out_dtype=dt, workspace=ws)
    torch.cuda.synchronize()
    kvrq.device_status()
    xref = tq.prod_dequantize(ref["words"], ref["signs_words"], g64, n64, pi64, T64, c64, bits, d)
    _rows_close(to_f64(xh), xref, XHAT_RTOL[dt])


def test_zero_rows_tiled():
    d, bits, dt = 256, 3, torch.float16
    pi64, c64, T64, pi_d, c_d, T_d = _params(d, bits, dt)
    x = _input(300, d, dt, seed=9)
    x[[0, 131, 299]] = 0
    codes, norms, xhat = kvrq.tq_quantize_dequantize_mse(x, pi_d, c_d, bits)
    torch.cuda.synchronize()
    zc = ocodes.unpack(words_u32(codes)[[0, 131, 299]], d, bits)
    assert np.all(zc == (1 << (bits - 1)) - 1)  # y = 0 takes the lower middle code
    assert np.all(to_f64(xhat)[[0, 131, 299]] == 0) and np.all(to_f64(norms)[[0, 131, 299]] == 0)
    # prod: a zero row takes the lower middle codes, so its residual is -c_hat (gamma = ||c_hat||,
    # signs of -T c_hat), as in the oracle; its reconstruction is 0 through the zero norm
    pi64, c64, T64, pi_d, c_d, T_d = _params(d, bits - 1, dt)
    codes, signs, gammas, norms = kvrq.tq_quantize_prod(x, pi_d, T_d, c_d, bits)
    torch.cuda.synchronize()
    z = [0, 131, 299]
    ref = tq.prod_quantize(to_f64(x)[z], pi64, T64, c64, bits)
    assert np.allclose(to_f64(gammas)[z], ref["gammas"], rtol=1e-5)
    assert np.array_equal(words_u32(signs)[z], ref["signs_words"])
    xh = kvrq.tq_dequantize(codes, norms, d, pi_d, c_d, bits, signs=signs, gammas=gammas, T=T_d)
    assert np.all(to_f64(xh)[z] == 0)


@pytest.mark.parametrize("d,m,dt,n", [
    (128, 128, torch.float16, 300), (256, 256, torch.bfloat16, 1000), (192, 384, torch.float16, 77),
    (64, 128, torch.float32, 200), (1536, 1536, torch.float16, 140), (256, 128, torch.float32, 129),
])
def test_qjl_sketch(d, m, dt, n):
    r = synth.gaussian(n, d, seed=d + m, dtype=dt).cuda()
    tdt = torch.float16 if dt == torch.float32 else dt
    T_d = torch.from_numpy(params.qjl_matrix(m, d, 5)).to(tdt).cuda()
    signs, gammas = kvrq.qjl_sketch(r, T_d)
    torch.cuda.synchronize()
    kvrq.device_status()
    r64, T64 = to_f64(r), to_f64(T_d)
    ref = tq.qjl_sketch(r64, T64)
    assert np.allclose(to_f64(gammas), ref["gammas"], rtol=1e-5)
    gs = ocodes.unpack(words_u32(signs), m, 1)
    os_ = ocodes.unpack(ref["signs_words"], m, 1)
    cos = ref["p"] / (np.linalg.norm(T64, axis=1)[None, :] * np.linalg.norm(r64, axis=1)[:, None])
    diff = gs != os_
    assert np.all(np.abs(cos[diff]) < SIGN_MARGIN), "sign mismatch away from zero"


@pytest.mark.parametrize("d,dt,n", [(1536, torch.float16, 8253), (1024, torch.bfloat16, 12000),
                                    (256, torch.float16, 60001)])
def test_many_tiles_per_cta(d, dt, n):
    """Several tiles per CTA (the stage ring and the norm hand-off wrap many times): every row's
    norm, codes, gamma and sign against the oracle, for the MSE quantizer, TurboQuant-prod through
    row blocks of a small workspace, and the QJL sketch."""
    x = _input(n, d, dt, seed=d + n)
    x64 = to_f64(x)
    nrm64 = np.linalg.norm(x64, axis=1)
    pi64, c64, T64, pi_d, c_d, T_d = _params(d, 2, dt)
    codes, norms = kvrq.tq_quantize_mse(x, pi_d, c_d, 2)
    torch.cuda.synchronize()
    kvrq.device_status()
    assert np.allclose(to_f64(norms), nrm64, rtol=1e-5)
    ref = tq.mse_quantize(x64, pi64, c64, 2)
    compare_codes(words_u32(codes), ref, d, 2, c64)

    ws = torch.empty((kvrq.tq_workspace_bytes(2048, d),), dtype=torch.uint8, device="cuda")
    codes, signs, gammas, norms = kvrq.tq_quantize_prod(x, pi_d, T_d, c_d, 3, workspace=ws)
    torch.cuda.synchronize()
    kvrq.device_status()
    assert np.allclose(to_f64(norms), nrm64, rtol=1e-5)
    ref = tq.prod_quantize(x64, pi64, T64, c64, 3)
    nb, bad = compare_codes(words_u32(codes), ref, d, 2, c64)
    assert np.allclose(to_f64(gammas)[~bad], ref["gammas"][~bad], rtol=1e-4, atol=1e-7)
    compare_sketch_signs(words_u32(signs), ref, x64, pi64, T64, c64, skip_rows=bad)

    T_s = T_d.to(dt)  # the sketch takes T in the vectors' own 16-bit type
    signs, gammas = kvrq.qjl_sketch(x, T_s)
    torch.cuda.synchronize()
    kvrq.device_status()
    assert np.allclose(to_f64(gammas), nrm64, rtol=1e-5)
    Ts64 = to_f64(T_s)
    sk = tq.qjl_sketch(x64, Ts64)
    cos = sk["p"] / (np.linalg.norm(Ts64, axis=1)[None, :] * nrm64[:, None])
    diff = ocodes.unpack(words_u32(signs), d, 1) != ocodes.unpack(sk["signs_words"], d, 1)
    assert np.all(np.abs(cos[diff]) < SIGN_MARGIN), "sign mismatch away from zero"
