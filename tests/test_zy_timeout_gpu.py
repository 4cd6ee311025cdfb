"""The device time-out path, with no fault: the packed-score kernel's tile waits are limited to no polls
(kvrq_set_wait_limit(0)), so they give up while the first bulk copies are still landing. The kernel must drain its
own copies and tensor-core products, free its tensor memory and return; kvrq_device_status then reports
KVRQ_ETIMEOUT (and clears it), and the next launches, at the default limit, run correctly on the same context.
(Collected after the other GPU tests, which it must not disturb.)"""

import numpy as np
import pytest
import torch

import kv_cache_vector_rq_b200 as kvrq
from kv_cache_vector_rq_b200 import KvrqError, synth
from oracle import codebook, params

pytestmark = pytest.mark.gpu

D = 128


def _setup(heads=72, tokens=8192):
    pi = torch.from_numpy(params.rotation(D, 2)).to(torch.float16).cuda()
    T = torch.from_numpy(params.qjl_matrix(D, D, 3)).to(torch.float16).cuda()
    c = torch.from_numpy(codebook.lloyd_max(D, 2)[0].astype(np.float32)).cuda()
    k = synth.lognormal(heads * tokens, D, seed=3, dtype=torch.float16, device="cuda")
    codes, signs, gam, norms = kvrq.tq_quantize_prod(k, pi, T, c, 3)
    q = synth.gaussian(heads * 8, D, seed=4, dtype=torch.float16, device="cuda").view(heads, 8, D)
    args = (kvrq.TQ_PROD, q, codes.view(heads, tokens, -1), norms.view(heads, tokens), 3, tokens, c)
    kw = dict(pi=pi, T=T, signs=signs.view(heads, tokens, -1), gammas=gam.view(heads, tokens))
    return args, kw


def test_wait_runs_out_and_the_context_recovers():
    args, kw = _setup()
    ref = kvrq.kv_score_packed(*args, **kw)
    torch.cuda.synchronize()
    kvrq.device_status()  # nothing pending
    try:
        kvrq.lib().kvrq_set_wait_limit(0)
        kvrq.kv_score_packed(*args, **kw)
        torch.cuda.synchronize()  # the kernel returned: no hang, no fault
    finally:
        kvrq.lib().kvrq_set_wait_limit(-1)
    with pytest.raises(KvrqError) as e:
        kvrq.device_status()
    assert e.value.status == 5  # KVRQ_ETIMEOUT
    kvrq.device_status()  # read once, then cleared
    again = kvrq.kv_score_packed(*args, **kw)
    torch.cuda.synchronize()
    kvrq.device_status()
    assert torch.equal(again, ref)


def test_attention_copy_wait_runs_out_and_the_context_recovers():
    """The tensor-core attention kernel under the same zero limit: every warpgroup's first tile-copy wait gives
    up, the warpgroup writes nothing to tensor memory, waits (at the default limit) for the copy it issued and
    stops; the status reads KVRQ_ETIMEOUT once, and the next call reproduces the reference bit for bit."""
    heads, tokens = 16, 4096
    pi = torch.from_numpy(params.rotation(D, 2)).to(torch.float16).cuda()
    T = torch.from_numpy(params.qjl_matrix(D, D, 3)).to(torch.float16).cuda()
    ck = torch.from_numpy(codebook.lloyd_max(D, 2)[0].astype(np.float32)).cuda()
    cv = torch.from_numpy(codebook.lloyd_max(D, 3)[0].astype(np.float32)).cuda()
    rot = torch.from_numpy(params.rotors(D, 5).astype(np.float32)).cuda()
    k = synth.lognormal(heads * tokens, D, seed=6, dtype=torch.float16, device="cuda")
    v = synth.lognormal(heads * tokens, D, seed=7, dtype=torch.float16, device="cuda")
    kc, ks, kg, kn = kvrq.tq_quantize_prod(k, pi, T, ck, 3)
    vc, vn = kvrq.rq_quantize(v, rot, cv, 3)
    q = synth.gaussian(heads * 8, D, seed=8, dtype=torch.float16, device="cuda").view(heads, 8, D)
    assert kvrq.attention_uses_tensor_cores(kvrq.TQ_PROD, 3, 3, 8)

    def run():
        return kvrq.kv_attention_packed(kvrq.TQ_PROD, q, kc.view(heads, tokens, -1), kn.view(heads, tokens), 3,
                                        vc.view(heads, tokens, -1), vn.view(heads, tokens), 3, tokens, ck, rot, cv,
                                        pi=pi, T=T, k_signs=ks.view(heads, tokens, -1),
                                        k_gammas=kg.view(heads, tokens))

    ref = run()
    torch.cuda.synchronize()
    kvrq.device_status()
    try:
        kvrq.lib().kvrq_set_wait_limit(0)
        run()
        torch.cuda.synchronize()  # the kernel returned: no hang, no fault
    finally:
        kvrq.lib().kvrq_set_wait_limit(-1)
    with pytest.raises(KvrqError) as e:
        kvrq.device_status()
    assert e.value.status == 5  # KVRQ_ETIMEOUT
    kvrq.device_status()
    again = run()
    torch.cuda.synchronize()
    kvrq.device_status()
    assert torch.equal(again, ref)
