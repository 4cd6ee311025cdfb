"""Decode-step append: one new vector per cache row quantized into its slot (GPU)."""

import numpy as np
import pytest
import torch

import kv_cache_vector_rq_b200 as kvrq
from kv_cache_vector_rq_b200 import synth
from oracle import codebook, params, rq, tq
from tests.parity import compare_codes, compare_sketch_signs, to_f64, words_u32

pytestmark = pytest.mark.gpu

D = 128
CANARY = 0x13579BDF


@pytest.mark.parametrize("method,bits", [("rq", 3), ("tq_mse", 3), ("tq_prod", 3), ("rq", 2), ("tq_prod", 4)])
def test_append_matches_plain_quantize_and_touches_only_the_slot(method, bits):
    rows, t_max, slot = 72, 50, 17
    dt = torch.bfloat16 if method == "tq_prod" else torch.float16
    x = synth.lognormal(rows, D, seed=11, dtype=dt).cuda()
    cb_bits = bits - 1 if method == "tq_prod" else bits
    c = torch.from_numpy(codebook.lloyd_max(D, cb_bits)[0].astype(np.float32)).cuda()
    rot = torch.from_numpy(params.rotors(D, 1).astype(np.float32)).cuda()
    pi = torch.from_numpy(params.rotation(D, 2)).to(dt).cuda()
    T = torch.from_numpy(params.qjl_matrix(D, D, 3)).to(torch.float16).cuda()
    ncode = 129 if method == "rq" else D
    W = kvrq.packed_words(ncode, cb_bits)
    codes = torch.full((rows, t_max, W), CANARY, dtype=torch.int32, device="cuda")
    norms = torch.full((rows, t_max), -5.0, device="cuda")
    gammas = torch.full((rows, t_max), -5.0, device="cuda")
    signs = torch.full((rows, t_max, 4), CANARY, dtype=torch.int32, device="cuda")
    mth = {"rq": kvrq.RQ_MSE, "tq_mse": kvrq.TQ_MSE, "tq_prod": kvrq.TQ_PROD}[method]
    kw = {"rq": dict(rotors=rot), "tq_mse": dict(pi=pi), "tq_prod": dict(pi=pi, T=T, signs=signs, gammas=gammas)}
    kvrq.kv_cache_append(mth, x, slot, bits, c, codes, norms, **kw[method])
    if method == "rq":
        rc, rn = kvrq.rq_quantize(x, rot, c, bits)
    elif method == "tq_mse":
        rc, rn = kvrq.tq_quantize_mse(x, pi, c, bits)
    else:
        rc, rs, rg, rn = kvrq.tq_quantize_prod(x, pi, T, c, bits)
    torch.cuda.synchronize()
    kvrq.device_status()
    assert torch.equal(codes[:, slot], rc) and torch.equal(norms[:, slot], rn)
    other = torch.ones(t_max, dtype=torch.bool)
    other[slot] = False
    assert torch.all(codes[:, other] == CANARY) and torch.all(norms[:, other] == -5.0)
    if method == "tq_prod":
        assert torch.equal(signs[:, slot], rs) and torch.equal(gammas[:, slot], rg)
        assert torch.all(signs[:, other] == CANARY) and torch.all(gammas[:, other] == -5.0)


@pytest.mark.parametrize("method", ["rq", "tq_mse", "tq_prod"])
def test_appended_slot_matches_oracle(method):
    """The slot written by the decode-step append against the oracle's quantization of the new vectors
    ("TurboQuant + RotorQuant", "Post-Prefill Quantization": one new K/V per step, quantized into the cache):
    codes by the boundary rule, norms (and gammas, QJL signs) as for the plain quantizers."""
    bits, rows, t_max, slot = 3, 600, 9, 5
    dt = torch.bfloat16 if method == "tq_prod" else torch.float16
    x = synth.lognormal(rows, D, seed=23, dtype=dt).cuda()
    cb_bits = bits - 1 if method == "tq_prod" else bits
    c32 = codebook.lloyd_max(D, cb_bits)[0].astype(np.float32)
    rot32 = params.rotors(D, 1).astype(np.float32)
    pi = torch.from_numpy(params.rotation(D, 2)).to(dt)
    T = torch.from_numpy(params.qjl_matrix(D, D, 3)).to(torch.float16)
    ncode = 129 if method == "rq" else D
    W = kvrq.packed_words(ncode, cb_bits)
    codes = torch.full((rows, t_max, W), CANARY, dtype=torch.int32, device="cuda")
    norms = torch.full((rows, t_max), -5.0, device="cuda")
    gammas = torch.full((rows, t_max), -5.0, device="cuda")
    signs = torch.full((rows, t_max, 4), CANARY, dtype=torch.int32, device="cuda")
    mth = {"rq": kvrq.RQ_MSE, "tq_mse": kvrq.TQ_MSE, "tq_prod": kvrq.TQ_PROD}[method]
    c_d = torch.from_numpy(c32).cuda()
    kw = {"rq": dict(rotors=torch.from_numpy(rot32).cuda()), "tq_mse": dict(pi=pi.cuda()),
          "tq_prod": dict(pi=pi.cuda(), T=T.cuda(), signs=signs, gammas=gammas)}
    kvrq.kv_cache_append(mth, x, slot, bits, c_d, codes, norms, **kw[method])
    torch.cuda.synchronize()
    kvrq.device_status()
    x64, c64, pi64 = to_f64(x), c32.astype(np.float64), pi.double().numpy()
    if method == "rq":
        ref = rq.quantize(x64, rot32.astype(np.float64), c64, bits)
    elif method == "tq_mse":
        ref = tq.mse_quantize(x64, pi64, c64, bits)
    else:
        ref = tq.prod_quantize(x64, pi64, T.double().numpy(), c64, bits)
    _, bad = compare_codes(words_u32(codes[:, slot]), ref, ncode, cb_bits, c64)
    assert np.allclose(to_f64(norms[:, slot]), ref["norms"], rtol=1e-5)
    if method == "tq_prod":
        g = to_f64(gammas[:, slot])
        assert np.allclose(g[~bad], ref["gammas"][~bad], rtol=1e-4, atol=1e-7)
        compare_sketch_signs(words_u32(signs[:, slot]), ref, x64, pi64, T.double().numpy(), c64, skip_rows=bad)
