"""The host-buffer RotorQuant roundtrip (rq_quantize_dequantize_host): rows copied in chunks through the device,
copy-in, kernel and copy-out of successive chunks overlapped on the library's streams. Its outputs must equal the
device call on the same rows bit for bit, for chunk counts that leave a ragged last chunk, strided host rows and
code rows, pageable host memory, and two calls in a row sharing one workspace ("TurboQuant + RotorQuant",
"Post-Prefill Quantization": a prefill cache quantized in bulk)."""

import numpy as np
import pytest
import torch

import kv_cache_vector_rq_b200 as kvrq
from kv_cache_vector_rq_b200 import synth
from oracle import codebook, params, rq
from tests.parity import compare_codes, to_f64, words_u32

pytestmark = pytest.mark.gpu


def _params(d, bits):
    rot = torch.from_numpy(params.rotors(d, 1).astype(np.float32)).cuda()
    c = torch.from_numpy(codebook.lloyd_max(d, bits)[0].astype(np.float32)).cuda()
    return rot, c


def _device_ref(x_host, rot, c, bits):
    codes, norms, xhat = kvrq.rq_quantize_dequantize(x_host.cuda(), rot, c, bits)
    torch.cuda.synchronize()
    return codes.cpu(), norms.cpu(), xhat.cpu()


@pytest.mark.parametrize("d,dt,n,chunk", [(128, torch.float16, 10000, 1024), (128, torch.bfloat16, 777, 32),
                                          (256, torch.float16, 3000, 256), (1536, torch.float16, 500, 64),
                                          (100, torch.float32, 999, 128)])
def test_host_roundtrip_equals_device_call(d, dt, n, chunk):
    bits = 3
    rot, c = _params(d, bits)
    x = synth.lognormal(n, d, seed=n + d, dtype=dt).pin_memory()
    ws = torch.empty(kvrq.host_workspace_bytes(d, bits, dt, chunk), dtype=torch.uint8, device="cuda")
    codes, norms, xhat = kvrq.rq_quantize_dequantize_host(x, rot, c, bits, ws)
    torch.cuda.synchronize()
    kvrq.device_status()
    rc, rn, rx = _device_ref(x, rot, c, bits)
    assert torch.equal(codes, rc) and torch.equal(norms, rn)
    iv = torch.int16 if x.element_size() == 2 else torch.int32
    assert torch.equal(xhat.view(iv), rx.view(iv))
    # and the oracle on a sample of the rows
    rows = np.unique(np.linspace(0, n - 1, 64).astype(int))
    rot64 = params.rotors(d, 1).astype(np.float32).astype(np.float64)
    c64 = codebook.lloyd_max(d, bits)[0].astype(np.float32).astype(np.float64)
    ref = rq.roundtrip(to_f64(x[rows]), rot64, c64, bits)
    compare_codes(words_u32(codes[rows]), ref, 3 * kvrq.rq_groups(d), bits, c64)


def test_strided_pageable_rows_and_back_to_back_calls():
    d, bits, n = 128, 2, 5000
    rot, c = _params(d, bits)
    base = synth.lognormal(n, d + 8, seed=3, dtype=torch.float16)  # pageable, rows of d + 8 elements
    x = base[:, :d]
    W = kvrq.packed_words(129, bits)
    codes = torch.full((n, W + 3), -1, dtype=torch.int32)[:, :W]  # code rows of W + 3 words
    xhat = torch.full((n, d + 16), 7.0, dtype=torch.float16)[:, :d]
    ws = torch.empty(kvrq.host_workspace_bytes(d, bits, torch.float16, 512), dtype=torch.uint8, device="cuda")
    kvrq.rq_quantize_dequantize_host(x, rot, c, bits, ws, codes=codes, xhat=xhat)
    # a second call with other rows and the same workspace, queued right behind the first
    y = synth.lognormal(300, d, seed=4, dtype=torch.float16).pin_memory()
    c2, n2, x2 = kvrq.rq_quantize_dequantize_host(y, rot, c, bits, ws)
    torch.cuda.synchronize()
    kvrq.device_status()
    rc, rn, rx = _device_ref(x.contiguous(), rot, c, bits)
    assert torch.equal(codes, rc) and torch.equal(xhat.view(torch.int16), rx.view(torch.int16))
    # the columns past each row are untouched
    assert torch.all(xhat.as_strided((n, 16), (d + 16, 1), d) == 7.0)
    assert torch.all(codes.as_strided((n, 3), (W + 3, 1), W) == -1)
    yc, yn, yx = _device_ref(y, rot, c, bits)
    assert torch.equal(c2, yc) and torch.equal(n2, yn) and torch.equal(x2.view(torch.int16), yx.view(torch.int16))
