"""GPU parity of the RotorQuant kernels against the float64 oracle (through the C ABI)."""

import numpy as np
import pytest
import torch

import kv_cache_vector_rq_b200 as kvrq
from kv_cache_vector_rq_b200 import synth
from oracle import codebook, codes as ocodes, params, rq
from tests.parity import compare_codes, compare_floats, to_f64, words_u32

pytestmark = pytest.mark.gpu

DT = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}
CANARY = 0x5A5A5A5A


def _params(d, bits, seed=1):
    """Oracle-generated parameters, rounded to the device types; the oracle gets the rounded values."""
    rot = params.rotors(d, seed).astype(np.float32)
    c, _, _ = codebook.lloyd_max(d, bits)
    c = c.astype(np.float32)
    return (rot.astype(np.float64), c.astype(np.float64),
            torch.from_numpy(rot).cuda(), torch.from_numpy(c).cuda())


def _check_roundtrip(x_dev, bits, seed=1, sample=None, check_dequant=True):
    n, d = x_dev.shape
    rot64, c64, rot_d, c_d = _params(d, bits, seed)
    codes, norms, xhat = kvrq.rq_quantize_dequantize(x_dev, rot_d, c_d, bits)
    torch.cuda.synchronize()
    kvrq.device_status()
    rows = np.arange(n) if sample is None else sample
    x64 = to_f64(x_dev[torch.as_tensor(rows, device="cuda")])
    ref = rq.roundtrip(x64, rot64, c64, bits)
    G = kvrq.rq_groups(d)
    w = words_u32(codes)[rows]
    nb, bad_rows = compare_codes(w, ref, 3 * G, bits, c64)
    assert np.allclose(to_f64(norms)[rows], ref["norms"], rtol=1e-5, atol=0)
    compare_floats(to_f64(xhat)[rows], ref["xhat"], x_dev.dtype, ref["norms"], skip_rows=bad_rows)
    if check_dequant:
        # dequantize of the GPU codes reproduces the fused output bit for bit
        xd = kvrq.rq_dequantize(codes, norms, d, rot_d, c_d, bits, out_dtype=x_dev.dtype)
        assert torch.equal(xd.view(torch.int16 if x_dev.element_size() == 2 else torch.int32),
                           xhat.view(torch.int16 if x_dev.element_size() == 2 else torch.int32))
        # quantize-only gives the same codes and norms
        c2, n2 = kvrq.rq_quantize(x_dev, rot_d, c_d, bits)
        assert torch.equal(c2, codes) and torch.equal(n2, norms)
    return nb, ref, xhat


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_config1_fp32_gaussian(bits):
    x = synth.gaussian(1024, 128, seed=0, dtype=torch.float32).cuda()
    nb, ref, xhat = _check_roundtrip(x, bits)
    assert nb <= 2
    if bits == 3:
        xf = to_f64(x)
        u = xf / np.linalg.norm(xf, axis=1, keepdims=True)
        xh = to_f64(xhat) / np.linalg.norm(xf, axis=1, keepdims=True)
        mse = np.mean(np.sum((u - xh) ** 2, axis=1))
        assert abs(mse - 0.034) < 0.003


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_config2_full_size_fp16_sampled(bits):
    x = synth.lognormal(65536, 128, seed=0, dtype=torch.float16).cuda()
    sample = np.sort(np.random.default_rng(bits).choice(65536, 2048, replace=False))
    sample = np.unique(np.concatenate([sample, [0, 127, 128, 65535]]))
    nb, _, _ = _check_roundtrip(x, bits, sample=sample)
    assert nb <= 5


@pytest.mark.parametrize("dt", ["f16", "bf16", "f32"])
@pytest.mark.parametrize("n", [1, 5, 127, 128, 129, 3000])
def test_ragged_row_counts(dt, n):
    x = synth.lognormal(n, 128, seed=n, dtype=DT[dt]).cuda()
    _check_roundtrip(x, 3)


def test_zero_rows_and_extreme_norms():
    x = synth.gaussian(300, 128, seed=4, dtype=torch.float32)
    x[7] = 0.0
    x[8] *= 1e-3
    x[9] *= 1e3
    x[200] = 0.0
    xd = x.to(torch.float16).cuda()
    _, ref, xhat = _check_roundtrip(xd, 3)
    assert np.all(to_f64(xhat)[[7, 200]] == 0.0)


@pytest.mark.parametrize("d", [2, 3, 4, 5, 64, 100, 129, 256, 1536])
@pytest.mark.parametrize("bits", [1, 3, 4])
def test_general_dimensions(d, bits):
    x = synth.lognormal(517, d, seed=d, dtype=torch.float16).cuda()
    _check_roundtrip(x, bits)


@pytest.mark.parametrize("d,dt,n", [(4096, torch.float16, 300), (4096, torch.bfloat16, 130), (1536, torch.bfloat16, 333),
                                    (8, torch.float16, 5000), (24, torch.float32, 1000), (2048, torch.float32, 77)])
def test_general_dimensions_bulk_rows(d, dt, n):
    # rows that start 16-byte aligned go through the bulk-copy kernel (several row blocks per warp)
    x = synth.lognormal(n, d, seed=d + n, dtype=dt).cuda()
    _check_roundtrip(x, 3)


def test_general_bulk_rows_strided():
    # 16-byte aligned but not contiguous rows: per-row copies
    base = synth.lognormal(400, 264, seed=3, dtype=torch.float16).cuda()
    _check_roundtrip(base[:, :256], 2)


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
@pytest.mark.parametrize("dt", ["f16", "bf16"])
def test_ring_sizes(dt, bits):
    # 160,033 rows: every warp has two 32-row sub-tiles or more (16-warp CTAs, 14 at b = 4), so the
    # quantizing modes take the ring of half-tile boxes; dequantize (never the ring) must reproduce the
    # fused x_hat bit for bit
    n = 160033
    x = synth.lognormal(n, 128, seed=bits + 7, dtype=DT[dt]).cuda()
    sample = np.unique(np.concatenate([np.random.default_rng(bits).choice(n, 1536, replace=False),
                                       [0, 31, 32, 4095, n - 33, n - 1]]))
    nb, _, _ = _check_roundtrip(x, bits, sample=np.sort(sample))
    assert nb <= 5


@pytest.mark.parametrize("bits", [2, 4])
def test_d256_bf16_row_kernel(bits):
    x = synth.lognormal(1000, 256, seed=bits, dtype=torch.bfloat16).cuda()
    _check_roundtrip(x, bits)


def test_general_dimension_4096_fp32():
    x = synth.gaussian(200, 4096, seed=9, dtype=torch.float32).cuda()
    _check_roundtrip(x, 3)


def test_strided_input_and_padded_code_rows():
    base = synth.lognormal(700, 136, seed=5, dtype=torch.float16).cuda()
    x = base[:, :128]  # ldx = 136: rows still 16-byte aligned (row kernel)
    bits = 3
    rot64, c64, rot_d, c_d = _params(128, bits)
    codes = torch.full((700, 16), CANARY, dtype=torch.int32, device="cuda")
    norms = torch.empty(700, dtype=torch.float32, device="cuda")
    xhat_buf = torch.full((700, 136), 7.0, dtype=torch.float16, device="cuda")
    xhat = xhat_buf[:, :128]
    kvrq.rq_quantize_dequantize(x, rot_d, c_d, bits, codes=codes, norms=norms, xhat=xhat)
    torch.cuda.synchronize()
    ref = rq.roundtrip(to_f64(x), rot64, c64, bits)
    _, bad = compare_codes(words_u32(codes[:, :13]), ref, 129, bits, c64)
    assert torch.all(codes[:, 13:] == CANARY)
    assert torch.all(xhat_buf[:, 128:] == 7.0)
    compare_floats(to_f64(xhat), ref["xhat"], torch.float16, ref["norms"], skip_rows=bad)
    # an unaligned stride takes the general kernel
    base2 = synth.lognormal(300, 129, seed=6, dtype=torch.float16).cuda()
    _check_roundtrip(base2[:, :128], bits)


def test_dequantize_oracle_codes():
    # dequantize codes produced by the oracle, independently of the GPU quantizer
    bits, n, d = 3, 999, 128
    rot64, c64, rot_d, c_d = _params(d, bits)
    x = synth.lognormal(n, d, seed=12, dtype=torch.float32).numpy().astype(np.float64)
    ref = rq.roundtrip(x, rot64, c64, bits)
    codes = torch.from_numpy(ref["words"].astype(np.int64).astype(np.int32)).cuda()
    norms = torch.from_numpy(ref["norms"].astype(np.float32)).cuda()
    # the oracle's x_hat from float32-rounded norms
    xref = rq.dequantize(ref["words"], ref["norms"].astype(np.float32).astype(np.float64), rot64, c64, bits, d)
    for dt in (torch.float32, torch.float16, torch.bfloat16):
        xh = kvrq.rq_dequantize(codes, norms, d, rot_d, c_d, bits, out_dtype=dt)
        torch.cuda.synchronize()
        compare_floats(to_f64(xh), xref, dt, ref["norms"])


def test_output_canaries_untouched_on_ragged_tail():
    n, bits = 200, 2
    x = synth.lognormal(n, 128, seed=3, dtype=torch.float16).cuda()
    rot64, c64, rot_d, c_d = _params(128, bits)
    W = kvrq.packed_words(129, bits)
    codes_buf = torch.full((n + 2, W), CANARY, dtype=torch.int32, device="cuda")
    norms_buf = torch.full((n + 2,), -1.0, dtype=torch.float32, device="cuda")
    xh_buf = torch.full((n + 2, 128), -3.0, dtype=torch.float16, device="cuda")
    kvrq.rq_quantize_dequantize(x, rot_d, c_d, bits, codes=codes_buf[1:n + 1], norms=norms_buf[1:n + 1],
                                xhat=xh_buf[1:n + 1])
    torch.cuda.synchronize()
    assert torch.all(codes_buf[0] == CANARY) and torch.all(codes_buf[n + 1] == CANARY)
    assert norms_buf[0].item() == -1.0 and norms_buf[n + 1].item() == -1.0
    assert torch.all(xh_buf[0] == -3.0) and torch.all(xh_buf[n + 1] == -3.0)
    kvrq.device_status()


@pytest.mark.parametrize("d,bits,dt", [(264, 2, torch.float16), (384, 3, torch.bfloat16), (1000, 3, torch.float16),
                                       (1000, 1, torch.bfloat16), (3072, 4, torch.float16), (4608, 3, torch.float16),
                                       (4608, 2, torch.bfloat16)])
def test_run_lengths(d, bits, dt):
    """16-bit rows of d > 256 (a multiple of 8) take the warp-per-row kernel whose lanes own contiguous runs
    of 8, 16, 24 or 48 groups: lanes past the last group, a zero-padded last group (d = 1000), and the
    largest d the run table and row buffers fit (4608)."""
    x = synth.lognormal(97, d, seed=d + bits, dtype=dt).cuda()
    _check_roundtrip(x, bits)


@pytest.mark.parametrize("dt", [torch.float16, torch.bfloat16])
def test_run_zero_rows_and_extreme_norms(dt):
    d = 1536
    x = synth.lognormal(64, d, seed=4, dtype=torch.float32)
    x[3] = 0.0
    if dt == torch.bfloat16:
        x[5] *= 1e30  # norms beyond fp32's square range: the power-of-two prescale
        x[6] *= 1e-30
    _, _, xhat = _check_roundtrip(x.to(dt).cuda(), 3)
    assert np.all(to_f64(xhat)[3] == 0.0)
