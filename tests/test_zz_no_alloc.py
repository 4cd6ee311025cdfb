"""tq_quantize_prod_noalloc: the prod quantizer run through the library's static
scratch. It must give the bits of tq_quantize_prod with a caller workspace, on
consecutive calls, without allocating device memory. This file is collected
last, so the check also holds after every other test has run."""

import numpy as np
import pytest
import torch

import kv_cache_vector_rq_b200 as kvrq
from kv_cache_vector_rq_b200 import synth
from oracle import codebook, params

P = 0x10000  # a fake, 16-byte aligned device address: validation fails before it is used


def test_noalloc_rejects_oversize_before_any_launch():
    lib = kvrq.lib()
    EINVAL, EUNSUP = 1, 2
    d = 16384  # one 128-row block needs 128 * (4 d + d / 32) bytes > 8 MiB

    def call(d=d, n=10, dt=1, bits=3, codes=P, ldc=None):
        W = -(-d * (bits - 1) // 32)
        return lib.tq_quantize_prod_noalloc(None, P, dt, n, d, d, P, P, d, P, bits, codes,
                                            W if ldc is None else ldc, P, d // 32, P, P)

    assert call() == EUNSUP
    assert "static scratch" in lib.kvrq_last_error_string().decode()
    assert call(d=8192, codes=None) == EINVAL  # a block fits; the missing output is reported
    assert call(d=192) == EUNSUP
    assert call(n=0, d=8192) == 0


@pytest.mark.gpu
@pytest.mark.parametrize("d,dt,n,bits", [(256, torch.float16, 3000, 3), (4096, torch.bfloat16, 1100, 2),
                                         (128, torch.float32, 20000, 4), (128, torch.float16, 500, 3)])
def test_noalloc_matches_workspace_call_twice(d, dt, n, bits):
    pdt = torch.float16 if dt == torch.float32 else dt
    pi = torch.from_numpy(params.rotation(d, 2)).to(pdt).cuda()
    T = torch.from_numpy(params.qjl_matrix(d, d, 3)).to(torch.float16).cuda()
    c = torch.from_numpy(codebook.lloyd_max(d, bits - 1)[0].astype(np.float32)).cuda()
    if dt == torch.float32:
        x = synth.gaussian(n, d, seed=7, dtype=dt).cuda()
    else:
        x = synth.lognormal(n, d, seed=7, dtype=dt, outliers=()).cuda()
    ref = kvrq.tq_quantize_prod(x, pi, T, c, bits)  # caller-owned workspace
    torch.cuda.synchronize()
    outs = []
    for _ in range(2):  # outputs allocated up front, so the calls themselves run with no allocation around
        W = kvrq.packed_words(d, bits - 1)
        outs.append((torch.empty((n, W), dtype=torch.int32, device="cuda"),
                     torch.empty((n,), dtype=torch.float32, device="cuda"),
                     torch.empty((n, d // 32), dtype=torch.int32, device="cuda"),
                     torch.empty((n,), dtype=torch.float32, device="cuda")))
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    for codes, norms, signs, gammas in outs:
        kvrq.tq_quantize_prod_noalloc(x, pi, T, c, bits, codes=codes, norms=norms, signs=signs, gammas=gammas)
    torch.cuda.synchronize()
    kvrq.device_status()
    assert torch.cuda.mem_get_info()[0] == free0
    for codes, norms, signs, gammas in outs:
        assert torch.equal(codes, ref[0]) and torch.equal(signs, ref[1])
        assert torch.equal(gammas, ref[2]) and torch.equal(norms, ref[3])
