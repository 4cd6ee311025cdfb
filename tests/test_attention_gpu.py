"""GPU parity of decode attention from a packed KV cache against the oracle.

Tolerance, by the kernel that runs (kvrq.attention_uses_tensor_cores):
* CUDA-core kernel: fp32 from the same rounded parameters (Pi and T in fp16, rotors
  and centroids in fp32) that the oracle reads as float64. Logit errors are ~1e-6
  relative, so the softmax weights agree to ~1e-6; the weighted sum of up to a few
  thousand fp32 terms adds at most ~sqrt(T) * 2^-24 * max|v_hat| in the typical
  case. Every output element must lie within 1e-3 * (largest |output| of its row)
  + 1e-5 * max|v_hat|: the 1e-3 relative bound of the fp32 path with an absolute
  floor for that accumulation.
* Tensor-core kernel: the rotated queries, T q', the centroids and the softmax
  weights enter the MMAs as fp16; a CPU restatement of that arithmetic
  (tests/test_attention_tolerance.py) reaches 1-2e-3 of the row's largest output, so
  the bound is 1e-2 of it (the tensor-core paths' relative bound) with the same floor.
"""

import numpy as np
import pytest
import torch

import kv_cache_vector_rq_b200 as kvrq
from kv_cache_vector_rq_b200 import synth
from oracle import attention, codebook, params, rq, tq
from tests.parity import attention_tolerance, random_words

pytestmark = pytest.mark.gpu

D = 128
METHODS = {"rq": kvrq.RQ_MSE, "tq_mse": kvrq.TQ_MSE, "tq_prod": kvrq.TQ_PROD}


def _params(k_method, k_bits, v_bits):
    cb = k_bits - 1 if k_method == "tq_prod" else k_bits
    kc = codebook.lloyd_max(D, cb)[0].astype(np.float32).astype(np.float64)
    vc = codebook.lloyd_max(D, v_bits)[0].astype(np.float32).astype(np.float64)
    pi = torch.from_numpy(params.rotation(D, 2)).to(torch.float16)
    T = torch.from_numpy(params.qjl_matrix(D, D, 3)).to(torch.float16)
    kp = {"centroids": kc, "rotors": params.rotors(D, 1).astype(np.float32).astype(np.float64),
          "Pi": pi.double().numpy(), "T": T.double().numpy()}
    vp = {"centroids": vc, "rotors": params.rotors(D, 4).astype(np.float32).astype(np.float64)}
    return kp, vp, pi, T


def _quantized_cache(k_method, k_bits, v_bits, n_heads, t_max, seed):
    """Keys and values quantized by the oracle from seeded synthetic KV rows."""
    kp, vp, pi, T = _params(k_method, k_bits, v_bits)
    keys = {"words": [], "norms": [], "signs_words": [], "gammas": []}
    values = {"words": [], "norms": []}
    for h in range(n_heads):
        k = synth.lognormal(t_max, D, seed=seed * 100 + h, dtype=torch.float32).numpy().astype(np.float64)
        v = synth.lognormal(t_max, D, seed=seed * 100 + 50 + h, dtype=torch.float32).numpy().astype(np.float64)
        if k_method == "rq":
            qq = rq.quantize(k, kp["rotors"], kp["centroids"], k_bits)
        elif k_method == "tq_mse":
            qq = tq.mse_quantize(k, kp["Pi"], kp["centroids"], k_bits)
        else:
            qq = tq.prod_quantize(k, kp["Pi"], kp["T"], kp["centroids"], k_bits)
            keys["signs_words"].append(qq["signs_words"])
            keys["gammas"].append(qq["gammas"].astype(np.float32).astype(np.float64))
        keys["words"].append(qq["words"])
        keys["norms"].append(qq["norms"].astype(np.float32).astype(np.float64))
        vq = rq.quantize(v, vp["rotors"], vp["centroids"], v_bits)
        values["words"].append(vq["words"])
        values["norms"].append(vq["norms"].astype(np.float32).astype(np.float64))
    keys = {kk: np.stack(v) for kk, v in keys.items() if v}
    values = {kk: np.stack(v) for kk, v in values.items()}
    return keys, kp, values, vp, pi, T


def _random_words(g, shape, n_codes, bits):
    """Uniformly random packed code rows (unused high bits of the last word zero)."""
    W = -(-n_codes * bits // 32)
    w = g.integers(0, 1 << 32, size=shape + (W,), dtype=np.uint64).astype(np.uint32)
    spare = W * 32 - n_codes * bits
    if spare:
        w[..., -1] &= np.uint32((1 << (32 - spare)) - 1)
    return w


def _random_cache(k_method, k_bits, v_bits, n_heads, t_max, seed):
    """Any code pattern is a valid cache: seeded random codes, norms and gammas."""
    kp, vp, pi, T = _params(k_method, k_bits, v_bits)
    g = np.random.default_rng(seed)
    cb = k_bits - 1 if k_method == "tq_prod" else k_bits
    nck = 129 if k_method == "rq" else D
    keys = {"words": _random_words(g, (n_heads, t_max), nck, cb),
            "norms": np.exp(0.5 * g.standard_normal((n_heads, t_max))).astype(np.float32).astype(np.float64)}
    if k_method == "tq_prod":
        keys["signs_words"] = _random_words(g, (n_heads, t_max), D, 1)
        keys["gammas"] = (0.3 * g.random((n_heads, t_max))).astype(np.float32).astype(np.float64)
    values = {"words": _random_words(g, (n_heads, t_max), 129, v_bits),
              "norms": np.exp(0.5 * g.standard_normal((n_heads, t_max))).astype(np.float32).astype(np.float64)}
    return keys, kp, values, vp, pi, T


def _dev_words(w):
    return torch.from_numpy(np.ascontiguousarray(np.asarray(w).astype(np.int64).astype(np.int32))).cuda()


def _dev_f32(a):
    return torch.from_numpy(np.ascontiguousarray(np.asarray(a, dtype=np.float32))).cuda()


def _run(k_method, k_bits, v_bits, keys, kp, values, vp, pi, T, q, n_tokens, scale, out_dtype=None):
    kw = {}
    if k_method == "rq":
        kw["k_rotors"] = _dev_f32(kp["rotors"])
    else:
        kw["pi"] = pi.cuda()
    if k_method == "tq_prod":
        kw.update(T=T.cuda(), k_signs=_dev_words(keys["signs_words"]), k_gammas=_dev_f32(keys["gammas"]))
    out = kvrq.kv_attention_packed(METHODS[k_method], q.cuda(), _dev_words(keys["words"]), _dev_f32(keys["norms"]),
                                   k_bits, _dev_words(values["words"]), _dev_f32(values["norms"]), v_bits, n_tokens,
                                   _dev_f32(kp["centroids"]), _dev_f32(vp["rotors"]), _dev_f32(vp["centroids"]),
                                   scale=scale, out_dtype=out_dtype, **kw)
    torch.cuda.synchronize()
    kvrq.device_status()
    return out.double().cpu().numpy()


def _rel(k_method, k_bits, v_bits, group):
    return 1e-2 if kvrq.attention_uses_tensor_cores(METHODS[k_method], k_bits, v_bits, group) else 1e-3


def _check(k_method, k_bits, v_bits, keys, kp, values, vp, q, n_tokens, scale, got, heads, rel=None):
    qf = q.double().numpy()
    if rel is None:
        rel = _rel(k_method, k_bits, v_bits, q.shape[1])
    for h in heads:
        kh = {kk: v[h:h + 1, :n_tokens] for kk, v in keys.items()}
        vh = {kk: v[h:h + 1, :n_tokens] for kk, v in values.items()}
        ref = attention.decode(k_method, qf[h], kh, kp, k_bits, vh, vp, v_bits, scale)  # [group, d]
        vmax = np.abs(attention.values_hat(vh, vp, v_bits, D)).max()
        tol = attention_tolerance(ref, vmax, rel)
        err = np.abs(got[h] - ref)
        assert np.all(err <= tol), "head %d: max excess %g (max err %g)" % (h, float((err - tol).max()), err.max())


@pytest.mark.parametrize("k_method,k_bits,v_bits", [("rq", 3, 3), ("tq_mse", 3, 3), ("tq_prod", 3, 3),
                                                    ("tq_prod", 2, 2), ("rq", 4, 4), ("tq_mse", 1, 2),
                                                    ("tq_prod", 4, 1)])
@pytest.mark.parametrize("group,n_heads,n_tokens,t_max", [(8, 3, 1000, 1024), (4, 2, 1, 8), (16, 2, 600, 640),
                                                          (1, 3, 257, 300)])
def test_attention_matches_oracle(k_method, k_bits, v_bits, group, n_heads, n_tokens, t_max):
    keys, kp, values, vp, pi, T = _quantized_cache(k_method, k_bits, v_bits, n_heads, t_max, seed=k_bits + group)
    q = (2.0 * torch.randn((n_heads, group, D), generator=torch.Generator().manual_seed(7))).to(torch.float16)
    scale = 1.0 / np.sqrt(D)
    got = _run(k_method, k_bits, v_bits, keys, kp, values, vp, pi, T, q, n_tokens, scale)
    _check(k_method, k_bits, v_bits, keys, kp, values, vp, q, n_tokens, scale, got, range(n_heads))


@pytest.mark.parametrize("k_method,n_heads,n_tok", [("tq_prod", 64, 20000), ("rq", 128, 8000)])
def test_attention_many_chunks_and_sub_chunks(k_method, n_heads, n_tok):
    """Enough heads x tokens for 512-token chunks: two 256-token sub-chunks per CTA, so the
    running max and sum are rescaled inside a CTA, and 40 (16) chunks merged per query row,
    the last one ragged. Random codes; the first and last heads are checked against the
    oracle."""
    group, k_bits, v_bits = 8, 3, 3
    keys, kp, values, vp, pi, T = _random_cache(k_method, k_bits, v_bits, n_heads, n_tok, seed=21)
    q = (3.0 * torch.randn((n_heads, group, D), generator=torch.Generator().manual_seed(8))).to(torch.bfloat16)
    scale = 1.0 / np.sqrt(D)
    got = _run(k_method, k_bits, v_bits, keys, kp, values, vp, pi, T, q, n_tok, scale)
    _check(k_method, k_bits, v_bits, keys, kp, values, vp, q, n_tok, scale, got, (0, n_heads - 1))


def test_attention_bf16_output_and_sharp_softmax():
    """A large logit scale makes the weights nearly one-hot (exercising the max subtraction);
    the output is written as bf16, compared at bf16 resolution."""
    keys, kp, values, vp, pi, T = _quantized_cache("tq_mse", 3, 3, 2, 500, seed=3)
    q = torch.randn((2, 8, D), generator=torch.Generator().manual_seed(2)).to(torch.float16)
    got = _run("tq_mse", 3, 3, keys, kp, values, vp, pi, T, q, 500, 2.0, out_dtype=torch.bfloat16)
    _check("tq_mse", 3, 3, keys, kp, values, vp, q, 500, 2.0, got, (0, 1), rel=1e-2)


# ---------------------------------------------------------------- tensor-core kernel

def test_tensor_core_path_selection():
    assert kvrq.attention_uses_tensor_cores(kvrq.TQ_PROD, 3, 3, 8)
    assert not kvrq.attention_uses_tensor_cores(kvrq.TQ_PROD, 3, 3, 9)  # the QJL rows need N = 2 x group
    assert kvrq.attention_uses_tensor_cores(kvrq.TQ_MSE, 3, 3, 16)
    assert kvrq.attention_uses_tensor_cores(kvrq.RQ_MSE, 3, 3, 16)
    assert not kvrq.attention_uses_tensor_cores(kvrq.RQ_MSE, 3, 4, 8)  # 4-bit values: CUDA cores
    assert not kvrq.attention_uses_tensor_cores(kvrq.TQ_MSE, 1, 3, 8)


@pytest.mark.parametrize("n_tokens", [1, 127, 128, 129, 255, 256, 257, 3001])
def test_tc_ragged_token_counts(n_tokens):
    """TurboQuant-prod 3-bit keys, RotorQuant 3-bit values, 8 query rows per KV head (the decode config):
    partial first tiles, exact tile multiples, one warpgroup without tiles, and a ragged last tile."""
    keys, kp, values, vp, pi, T = _quantized_cache("tq_prod", 3, 3, 3, n_tokens + 5, seed=n_tokens % 97)
    q = (2.0 * torch.randn((3, 8, D), generator=torch.Generator().manual_seed(n_tokens))).to(torch.float16)
    got = _run("tq_prod", 3, 3, keys, kp, values, vp, pi, T, q, n_tokens, 1.0 / np.sqrt(D))
    _check("tq_prod", 3, 3, keys, kp, values, vp, q, n_tokens, 1.0 / np.sqrt(D), got, range(3))


@pytest.mark.parametrize("k_method,k_bits,group", [("tq_prod", 3, 5), ("tq_prod", 4, 8), ("tq_mse", 2, 16),
                                                   ("tq_mse", 4, 3), ("rq", 2, 16), ("rq", 3, 7)])
def test_tc_key_methods(k_method, k_bits, group):
    keys, kp, values, vp, pi, T = _random_cache(k_method, k_bits, 3, 2, 2000, seed=group)
    q = (2.0 * torch.randn((2, group, D), generator=torch.Generator().manual_seed(group))).to(torch.bfloat16)
    assert kvrq.attention_uses_tensor_cores(METHODS[k_method], k_bits, 3, group)
    got = _run(k_method, k_bits, 3, keys, kp, values, vp, pi, T, q, 1999, 1.0 / np.sqrt(D))
    _check(k_method, k_bits, 3, keys, kp, values, vp, q, 1999, 1.0 / np.sqrt(D), got, (0, 1))


def test_tc_persistent_many_items():
    """More (head, chunk) work items than CTAs: every CTA rebuilds its query operand for several heads and
    keeps its stage ring and barrier phases across items."""
    n_heads, n_tok = 400, 1500
    keys, kp, values, vp, pi, T = _random_cache("tq_prod", 3, 3, n_heads, n_tok, seed=31)
    q = (3.0 * torch.randn((n_heads, 8, D), generator=torch.Generator().manual_seed(3))).to(torch.float16)
    got = _run("tq_prod", 3, 3, keys, kp, values, vp, pi, T, q, n_tok, 1.0 / np.sqrt(D))
    _check("tq_prod", 3, 3, keys, kp, values, vp, q, n_tok, 1.0 / np.sqrt(D), got, (0, 149, 150, 399))


def test_tc_padded_rows_take_per_thread_loads():
    """Code rows padded beyond their packed width (no contiguous tile blocks): every tile is loaded per
    thread instead of by bulk copy; same results."""
    n_heads, n_tok = 3, 1000
    keys, kp, values, vp, pi, T = _random_cache("tq_prod", 3, 3, n_heads, n_tok, seed=41)
    q = torch.randn((n_heads, 8, D), generator=torch.Generator().manual_seed(4)).to(torch.float16)
    pad = lambda w: np.concatenate([w, np.zeros(w.shape[:-1] + (3,), dtype=w.dtype)], axis=-1)
    kw = dict(pi=pi.cuda(), T=T.cuda(), k_signs=_dev_words(pad(keys["signs_words"])), k_gammas=_dev_f32(keys["gammas"]))
    out = kvrq.kv_attention_packed(kvrq.TQ_PROD, q.cuda(), _dev_words(pad(keys["words"])), _dev_f32(keys["norms"]), 3,
                                   _dev_words(pad(values["words"])), _dev_f32(values["norms"]), 3, n_tok,
                                   _dev_f32(kp["centroids"]), _dev_f32(vp["rotors"]), _dev_f32(vp["centroids"]), **kw)
    torch.cuda.synchronize()
    kvrq.device_status()
    got = out.double().cpu().numpy()
    _check("tq_prod", 3, 3, keys, kp, values, vp, q, n_tok, 1.0 / np.sqrt(D), got, range(n_heads))
    # and equal to the unpadded launch up to the order of the fp32 sums (the same tiles, the same MMAs)
    ref = _run("tq_prod", 3, 3, keys, kp, values, vp, pi, T, q, n_tok, 1.0 / np.sqrt(D))
    assert np.allclose(got, ref, rtol=0, atol=1e-6 * np.abs(ref).max())


@pytest.mark.parametrize("pi_dtype", [torch.float16, torch.bfloat16])
def test_query_rotation_with_two_byte_aligned_pi_and_T(pi_dtype):
    """Pi and T only 2-byte aligned (the call accepts that): the query rotation reads them element by element
    instead of in 16-byte vectors. The outputs match the oracle (fp16 Pi), and the aligned call within 2e-3 of
    the largest |output|: the two paths add the rotation's products in different orders, and a q' coordinate
    whose fp32 value moves by that rounding can round to a neighbouring fp16 value in the MMA operand (2^-11
    relative), which moves its logits and so the softmax weights by about that much."""
    n_heads, n_tok = 6, 700
    keys, kp, values, vp, pi, T = _random_cache("tq_prod", 3, 3, n_heads, n_tok, seed=53)
    q = (2.0 * torch.randn((n_heads, 8, D), generator=torch.Generator().manual_seed(5))).to(torch.float16)
    pi_buf = torch.zeros(D * D + 1, dtype=pi_dtype, device="cuda")
    pi_buf[1:] = pi.to(pi_dtype).cuda().reshape(-1)
    t_buf = torch.zeros(D * D + 1, dtype=torch.float16, device="cuda")
    t_buf[1:] = T.cuda().reshape(-1)
    pi_u, t_u = pi_buf[1:].view(D, D), t_buf[1:].view(D, D)
    assert pi_u.data_ptr() % 16 == 2 and t_u.data_ptr() % 16 == 2
    kw = dict(k_signs=_dev_words(keys["signs_words"]), k_gammas=_dev_f32(keys["gammas"]))
    args = (kvrq.TQ_PROD, q.cuda(), _dev_words(keys["words"]), _dev_f32(keys["norms"]), 3, _dev_words(values["words"]),
            _dev_f32(values["norms"]), 3, n_tok, _dev_f32(kp["centroids"]), _dev_f32(vp["rotors"]),
            _dev_f32(vp["centroids"]))
    out_u = kvrq.kv_attention_packed(*args, pi=pi_u, T=t_u, **kw)
    out_a = kvrq.kv_attention_packed(*args, pi=pi_u.clone(), T=t_u.clone(), **kw)
    torch.cuda.synchronize()
    kvrq.device_status()
    got = out_u.double().cpu().numpy()
    ref = out_a.double().cpu().numpy()
    if pi_dtype == torch.float16:
        _check("tq_prod", 3, 3, keys, kp, values, vp, q, n_tok, 1.0 / np.sqrt(D), got, range(n_heads))
    err = np.abs(got - ref).max() / np.abs(ref).max()
    assert err <= 2e-3, err
