"""GPU parity of RotorQuant in the pages' four-grade storage layout (172 codes per d = 128 vector:
per group the three vector components and the trivector component) against oracle/rq4.py, through
the C ABI ("TurboQuant + RotorQuant", "Parameter Efficiency", "FMA Count (d=128)")."""

import numpy as np
import pytest
import torch

import kv_cache_vector_rq_b200 as kvrq
from kv_cache_vector_rq_b200 import synth
from oracle import codebook, codes as ocodes, params, rq4
from tests.parity import compare_codes, compare_floats, device_words, to_f64, words_u32

pytestmark = pytest.mark.gpu

D = 128
G = 43
NC = 4 * G  # 172


def _params(bits, seed=1):
    rot = params.rotors(D, seed).astype(np.float32)
    c = codebook.lloyd_max(D, bits)[0].astype(np.float32)
    return rot.astype(np.float64), c.astype(np.float64), torch.from_numpy(rot).cuda(), torch.from_numpy(c).cuda()


def _decision(ref):
    """Decision values of the 172 codes: the vector components of the sandwich, and 0 for the trivector
    (stored as the code of exactly 0)."""
    mv = ref["mv"]
    comps = np.concatenate([mv[..., 1:4], np.zeros(mv.shape[:-1] + (1,))], axis=2)
    return comps.reshape(mv.shape[0], NC)


def _check(x, bits, rows=None):
    n = x.shape[0]
    rot64, c64, rot_d, c_d = _params(bits)
    codes, norms, xhat = kvrq.rq4_quantize_dequantize(x, rot_d, c_d, bits)
    torch.cuda.synchronize()
    kvrq.device_status()
    assert codes.shape == (n, kvrq.packed_words(NC, bits))
    rows = np.arange(n) if rows is None else rows
    idx = torch.as_tensor(rows, device="cuda")
    x64 = to_f64(x[idx])
    ref = rq4.quantize(x64, rot64, c64, bits)
    nb, bad = compare_codes(words_u32(codes[idx]), ref, NC, bits, c64, decision=_decision(ref))
    assert np.allclose(to_f64(norms[idx]), ref["norms"], rtol=1e-5)
    xref = rq4.dequantize(ref["words"], ref["norms"], rot64, c64, bits, D)
    compare_floats(to_f64(xhat[idx]), xref, x.dtype, ref["norms"], skip_rows=bad)
    # the trivector code of every group is the code of 0
    g = ocodes.unpack(words_u32(codes[idx]), NC, bits).reshape(len(rows), G, 4)
    assert np.all(g[..., 3] == (1 << (bits - 1)) - 1)
    # quantize-only and dequantize-only launches reproduce the fused one bit for bit
    c2, n2 = kvrq.rq4_quantize(x, rot_d, c_d, bits)
    xd = kvrq.rq4_dequantize(codes, norms, D, rot_d, c_d, bits, out_dtype=x.dtype)
    assert torch.equal(c2, codes) and torch.equal(n2, norms)
    iv = torch.int16 if x.element_size() == 2 else torch.int32
    assert torch.equal(xd.view(iv), xhat.view(iv))
    # same vector codes and x_hat as the three-code layout, bit for bit
    c3, n3, x3 = kvrq.rq_quantize_dequantize(x, rot_d, c_d, bits)
    v4 = ocodes.unpack(words_u32(codes), NC, bits).reshape(n, G, 4)[..., :3].reshape(n, 3 * G)
    assert np.array_equal(v4, ocodes.unpack(words_u32(c3), 3 * G, bits))
    assert torch.equal(x3.view(iv), xhat.view(iv)) and torch.equal(n3, norms)
    return nb


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_config1_fp32_gaussian(bits):
    x = synth.gaussian(1024, D, seed=0, dtype=torch.float32).cuda()
    assert _check(x, bits) <= 2


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_config2_full_size_fp16_sampled(bits):
    x = synth.lognormal(65536, D, seed=0, dtype=torch.float16).cuda()
    rows = np.unique(np.concatenate([np.random.default_rng(bits).choice(65536, 2048, replace=False),
                                     [0, 127, 128, 65535]]))
    assert _check(x, bits, rows) <= 5


@pytest.mark.parametrize("dt", [torch.float16, torch.bfloat16, torch.float32])
@pytest.mark.parametrize("n", [1, 31, 33, 3000])
def test_ragged_and_dtypes(dt, n):
    _check(synth.lognormal(n, D, seed=n, dtype=dt).cuda(), 3)


@pytest.mark.parametrize("bits", [1, 2, 4])
def test_ring_shape_large_launch(bits):
    # 200,000 rows is over two 32-row sub-tiles per warp of the GPU: the ring-buffered shape (b <= 2 in this
    # layout with 16-warp CTAs, b = 4 with 14; at b = 3 the code words of 16 warps do not fit)
    n = 200000
    x = synth.lognormal(n, D, seed=77, dtype=torch.float16).cuda()
    rows = np.unique(np.concatenate([np.random.default_rng(5).choice(n, 1500, replace=False), [0, n - 1]]))
    _check(x, bits, rows)


@pytest.mark.parametrize("bits", [2, 3])
def test_dequantize_of_oracle_and_random_codes(bits):
    """Any 172-code row is a valid input, trivector codes included (a pseudoscalar passes the inverse
    sandwich unchanged, so it never reaches x_hat): seeded random words against the oracle's dequantize."""
    rot64, c64, rot_d, c_d = _params(bits)
    g = np.random.default_rng(bits)
    n = 777
    W = kvrq.packed_words(NC, bits)
    w = g.integers(0, 1 << 32, size=(n, W), dtype=np.uint64).astype(np.uint32)
    spare = 32 * W - NC * bits
    if spare:
        w[:, -1] &= np.uint32((1 << (32 - spare)) - 1)
    nrm = np.exp(0.5 * g.standard_normal(n)).astype(np.float32)
    for dt in (torch.float32, torch.float16):
        xh = kvrq.rq4_dequantize(device_words(w), torch.from_numpy(nrm).cuda(), D, rot_d, c_d, bits, out_dtype=dt)
        torch.cuda.synchronize()
        ref = rq4.dequantize(w, nrm.astype(np.float64), rot64, c64, bits, D)
        compare_floats(to_f64(xh), ref, dt, nrm.astype(np.float64))


def test_unsupported_dimension_is_rejected():
    rot = torch.from_numpy(params.rotors(256, 1).astype(np.float32)).cuda()
    c = torch.from_numpy(codebook.lloyd_max(256, 3)[0].astype(np.float32)).cuda()
    x = torch.zeros((4, 256), dtype=torch.float16, device="cuda")
    with pytest.raises(kvrq.KvrqError):
        kvrq.rq4_quantize_dequantize(x, rot, c, 3)
