"""Decode-step append: one new vector per cache row quantized into its slot (GPU)."""

import numpy as np
import pytest
import torch

import kv_cache_vector_rq_b200 as kvrq
from kv_cache_vector_rq_b200 import synth
from oracle import codebook, params

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
