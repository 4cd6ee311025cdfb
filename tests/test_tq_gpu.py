"""GPU parity of the TurboQuant tensor-core kernels against the float64 oracle (through the C ABI)."""

import numpy as np
import pytest
import torch

import kv_cache_vector_rq_b200 as kvrq
from kv_cache_vector_rq_b200 import synth
from oracle import codebook, codes as ocodes, params, tq
from tests.parity import compare_codes, compare_sketch_signs, near_boundary, oracle_prod_inputs, to_f64, words_u32

pytestmark = pytest.mark.gpu

D = 128
# Tolerance of the reconstruction, normwise per row: the centroids enter the
# second tensor-core product rounded to the operand type (2^-11 relative for
# fp16, 2^-8 for bf16), plus the output's own rounding.
XHAT_RTOL = {torch.float16: 2e-3, torch.bfloat16: 1e-2}


def _params(bits_store, dt, seed=2):
    pi64 = params.rotation(D, seed)
    pi_d = torch.from_numpy(pi64).to(dt).cuda()
    c = codebook.lloyd_max(D, bits_store)[0].astype(np.float32)
    T_d = torch.from_numpy(params.qjl_matrix(D, D, seed + 1)).to(torch.float16).cuda()
    return (to_f64(pi_d), c.astype(np.float64), to_f64(T_d), pi_d, torch.from_numpy(c).cuda(), T_d)


def _rows_close(gpu, ref, rtol, skip=None):
    g = np.asarray(gpu, dtype=np.float64)
    r = np.asarray(ref, dtype=np.float64)
    keep = np.ones(len(g), bool) if skip is None else ~np.asarray(skip)
    rn = np.linalg.norm(r[keep], axis=1)
    err = np.linalg.norm(g[keep] - r[keep], axis=1)
    ok = rn > 0
    assert np.all(err[ok] <= rtol * rn[ok]), "normwise relative error %g" % (err[ok] / rn[ok]).max()
    assert np.all(err[~ok] == 0)


@pytest.mark.parametrize("dt", [torch.float16, torch.bfloat16])
@pytest.mark.parametrize("bits", [1, 2, 3, 4])
@pytest.mark.parametrize("n", [1, 300, 3000])
def test_mse_roundtrip(dt, bits, n):
    pi64, c64, _, pi_d, c_d, _ = _params(bits, dt)
    x = synth.lognormal(n, D, seed=n + bits, dtype=dt).cuda()
    codes, norms, xhat = kvrq.tq_quantize_dequantize_mse(x, pi_d, c_d, bits)
    torch.cuda.synchronize()
    kvrq.device_status()
    ref = tq.mse_quantize(to_f64(x), pi64, c64, bits)
    nb, bad = compare_codes(words_u32(codes), ref, D, bits, c64)
    assert np.allclose(to_f64(norms), ref["norms"], rtol=1e-5)
    xref = tq.mse_dequantize(ref["words"], ref["norms"], pi64, c64, bits, D)
    _rows_close(to_f64(xhat), xref, XHAT_RTOL[dt], skip=bad)
    # quantize-only and quantize-then-dequantize agree with the fused launch
    c2, n2 = kvrq.tq_quantize_mse(x, pi_d, c_d, bits)
    assert torch.equal(c2, codes) and torch.equal(n2, norms)
    xd = kvrq.tq_dequantize(codes, norms, D, pi_d, c_d, bits)
    assert torch.equal(xd, xhat)


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_mse_config2_full_size_sampled(bits):
    dt = torch.float16
    pi64, c64, _, pi_d, c_d, _ = _params(bits, dt)
    x = synth.lognormal(65536, D, seed=0, dtype=dt).cuda()
    codes, norms, xhat = kvrq.tq_quantize_dequantize_mse(x, pi_d, c_d, bits)
    torch.cuda.synchronize()
    rows = np.unique(np.concatenate([np.random.default_rng(bits).choice(65536, 2048, replace=False), [0, 65535]]))
    ref = tq.mse_quantize(to_f64(x)[rows], pi64, c64, bits)
    nb, bad = compare_codes(words_u32(codes)[rows], ref, D, bits, c64)
    xref = tq.mse_dequantize(ref["words"], ref["norms"], pi64, c64, bits, D)
    _rows_close(to_f64(xhat)[rows], xref, XHAT_RTOL[dt], skip=bad)


@pytest.mark.parametrize("dt", [torch.float16, torch.bfloat16])
@pytest.mark.parametrize("bits", [2, 3, 4])
@pytest.mark.parametrize("n", [77, 2000])
def test_prod_quantize_and_dequantize(dt, bits, n):
    pi64, c64, T64, pi_d, c_d, T_d = _params(bits - 1, dt)
    if dt == torch.bfloat16:
        x = synth.factor_keys(1, 1, n, D, seed=n, dtype=dt)[0, 0].contiguous().cuda()
    else:
        x = synth.lognormal(n, D, seed=n, dtype=dt).cuda()
    codes, signs, gammas, norms = kvrq.tq_quantize_prod(x, pi_d, T_d, c_d, bits)
    torch.cuda.synchronize()
    kvrq.device_status()
    ref = tq.prod_quantize(to_f64(x), pi64, T64, c64, bits)
    nb, bad = compare_codes(words_u32(codes), ref, D, bits - 1, c64)
    assert np.allclose(to_f64(norms), ref["norms"], rtol=1e-5)
    g = to_f64(gammas)
    assert np.allclose(g[~bad], ref["gammas"][~bad], rtol=1e-4, atol=1e-7)
    # signs: exact except where |T rho| is within the bound of the kernel's roundings
    compare_sketch_signs(words_u32(signs), ref, to_f64(x), pi64, T64, c64, skip_rows=bad)
    # dequantize the oracle's codes on the GPU, against the oracle's reconstruction of the same codes
    (oc, osg, og, on), g64, n64 = oracle_prod_inputs(ref)
    xh = kvrq.tq_dequantize(oc, on, D, pi_d, c_d, bits, signs=osg, gammas=og, T=T_d)
    torch.cuda.synchronize()
    xref = tq.prod_dequantize(ref["words"], ref["signs_words"], g64, n64, pi64, T64, c64, bits, D)
    _rows_close(to_f64(xh), xref, XHAT_RTOL[dt])


def test_zero_rows_tq():
    dt, bits = torch.float16, 3
    pi64, c64, T64, pi_d, c_d, T_d = _params(bits, dt)
    x = synth.lognormal(200, D, seed=5, dtype=dt)
    x[[3, 130]] = 0
    x = x.cuda()
    codes, norms, xhat = kvrq.tq_quantize_dequantize_mse(x, pi_d, c_d, bits)
    torch.cuda.synchronize()
    zc = ocodes.unpack(words_u32(codes)[[3, 130]], D, bits)
    assert np.all(zc == (1 << (bits - 1)) - 1)  # y = 0 takes the lower middle code
    assert np.all(to_f64(xhat)[[3, 130]] == 0) and np.all(to_f64(norms)[[3, 130]] == 0)


@pytest.mark.parametrize("dt", [torch.float16, torch.bfloat16])
def test_mse_many_tiles_per_cta(dt):
    """200,003 rows: every CTA of the d = 128 kernel takes five or six 128-row tiles, so both tile buffers
    and the loads issued during the previous tile are exercised, with a ragged last tile. Quantize-only and
    dequantize-only launches must reproduce the fused one bit for bit."""
    bits = 3
    n = 200003
    pi64, c64, _, pi_d, c_d, _ = _params(bits, dt)
    x = synth.lognormal(n, D, seed=12, dtype=dt).cuda()
    codes, norms, xhat = kvrq.tq_quantize_dequantize_mse(x, pi_d, c_d, bits)
    torch.cuda.synchronize()
    kvrq.device_status()
    rows = np.unique(np.concatenate([np.random.default_rng(9).choice(n, 3000, replace=False), [0, 127, 128, n - 1]]))
    ref = tq.mse_quantize(to_f64(x)[rows], pi64, c64, bits)
    nb, bad = compare_codes(words_u32(codes)[rows], ref, D, bits, c64)
    assert np.allclose(to_f64(norms)[rows], ref["norms"], rtol=1e-5)
    xref = tq.mse_dequantize(ref["words"], ref["norms"], pi64, c64, bits, D)
    _rows_close(to_f64(xhat)[rows], xref, XHAT_RTOL[dt], skip=bad)
    c2, n2 = kvrq.tq_quantize_mse(x, pi_d, c_d, bits)
    assert torch.equal(c2, codes) and torch.equal(n2, norms)
    xd = kvrq.tq_dequantize(codes, norms, D, pi_d, c_d, bits)
    torch.cuda.synchronize()
    assert torch.equal(xd, xhat)
