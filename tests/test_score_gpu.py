"""GPU parity of the packed-code score kernel against the oracle's direct scores."""

import numpy as np
import pytest
import torch

import kv_cache_vector_rq_b200 as kvrq
from kv_cache_vector_rq_b200 import synth
from oracle import codebook, params, rq, score, tq
from tests.parity import compare_scores, score_tolerance

pytestmark = pytest.mark.gpu

D = 128


def _keys(method, bits, n_heads, t_max, seed):
    """Oracle-quantized keys (the score kernel is tested on its own)."""
    g = np.random.default_rng(seed)
    cb_bits = bits - 1 if method == "tq_prod" else bits
    c = codebook.lloyd_max(D, cb_bits)[0].astype(np.float32).astype(np.float64)
    rot = params.rotors(D, 1).astype(np.float32).astype(np.float64)
    pi = torch.from_numpy(params.rotation(D, 2)).to(torch.float16)
    T = torch.from_numpy(params.qjl_matrix(D, D, 3)).to(torch.float16)
    p = {"centroids": c, "rotors": rot, "Pi": pi.double().numpy(), "T": T.double().numpy()}
    keys = {"words": [], "norms": [], "signs_words": [], "gammas": []}
    for h in range(n_heads):
        k = synth.lognormal(t_max, D, seed=seed * 100 + h, dtype=torch.float32).numpy().astype(np.float64)
        if method == "rq":
            qq = rq.quantize(k, rot, c, bits)
        elif method == "tq_mse":
            qq = tq.mse_quantize(k, p["Pi"], c, bits)
        else:
            qq = tq.prod_quantize(k, p["Pi"], p["T"], c, bits)
            keys["signs_words"].append(qq["signs_words"])
            keys["gammas"].append(qq["gammas"].astype(np.float32).astype(np.float64))
        keys["words"].append(qq["words"])
        keys["norms"].append(qq["norms"].astype(np.float32).astype(np.float64))
    keys = {kk: np.stack(v) for kk, v in keys.items() if v}
    return keys, p, pi.cuda(), T.cuda(), torch.from_numpy(c.astype(np.float32)).cuda(), torch.from_numpy(
        rot.astype(np.float32)).cuda()


def _dev_words(w):
    return torch.from_numpy(np.asarray(w).astype(np.int64).astype(np.int32)).cuda()


@pytest.mark.parametrize("method,bits", [("rq", 3), ("rq", 2), ("rq", 4), ("tq_mse", 3), ("tq_mse", 1),
                                         ("tq_mse", 4), ("tq_prod", 3), ("tq_prod", 2), ("tq_prod", 4)])
@pytest.mark.parametrize("group,n_heads,n_tokens,t_max", [(8, 4, 1000, 1000), (4, 3, 300, 384), (16, 2, 129, 200)])
def test_scores_match_oracle(method, bits, group, n_heads, n_tokens, t_max):
    if method == "tq_prod" and group > 32:
        pytest.skip("prod supports group <= 32")
    keys, p, pi_d, T_d, c_d, rot_d = _keys(method, bits, n_heads, t_max, seed=bits + group)
    q = torch.randn((n_heads, group, D), generator=torch.Generator().manual_seed(7)).to(torch.float16)
    mth = {"rq": kvrq.RQ_MSE, "tq_mse": kvrq.TQ_MSE, "tq_prod": kvrq.TQ_PROD}[method]
    kw = dict(rotors=rot_d) if method == "rq" else dict(pi=pi_d)
    if method == "tq_prod":
        kw.update(T=T_d, signs=_dev_words(keys["signs_words"]),
                  gammas=torch.from_numpy(keys["gammas"].astype(np.float32)).cuda())
    norms_d = torch.from_numpy(keys["norms"].astype(np.float32)).cuda()
    if method == "tq_prod":
        kw["gammas"] = kw["gammas"].contiguous()
    s = kvrq.kv_score_packed(mth, q.cuda(), _dev_words(keys["words"]), norms_d, bits, n_tokens, c_d, **kw)
    torch.cuda.synchronize()
    kvrq.device_status()
    got = s.double().cpu().numpy()
    qf = q.double().numpy()
    for h in range(n_heads):
        kh = {kk: v[h:h + 1, :n_tokens] for kk, v in keys.items()}
        ref = score.direct(method, qf[h], kh, p, bits)  # [group, n_tokens]
        compare_scores(got[h], ref, score_tolerance(method, qf[h], kh, p, bits), name="head %d" % h)


def test_score_of_gpu_quantized_keys_equals_dot_with_dequantized():
    # end to end on the device: TQ-prod keys quantized by the library, scores vs <q, x_hat>
    n_tok, bits = 777, 3
    pi = torch.from_numpy(params.rotation(D, 2)).to(torch.float16).cuda()
    T = torch.from_numpy(params.qjl_matrix(D, D, 3)).to(torch.float16).cuda()
    c = torch.from_numpy(codebook.lloyd_max(D, bits - 1)[0].astype(np.float32)).cuda()
    k = synth.factor_keys(1, 1, n_tok, D, seed=3, dtype=torch.float16)[0, 0].contiguous().cuda()
    codes, signs, gam, norms = kvrq.tq_quantize_prod(k, pi, T, c, bits)
    xh = kvrq.tq_dequantize(codes, norms, D, pi, c, bits, signs=signs, gammas=gam, T=T)
    q = torch.randn((1, 8, D), device="cuda").to(torch.float16)
    s = kvrq.kv_score_packed(kvrq.TQ_PROD, q, codes[None], norms[None], bits, n_tok, c, pi=pi, T=T,
                             signs=signs[None], gammas=gam[None])
    ref = (q[0].double() @ xh.double().T)
    tol = 1e-2 * q[0].double().norm(dim=1)[:, None] * norms.double()[None, :] + 1e-4
    assert torch.all((s[0].double() - ref).abs() <= tol)


def _random_words(g, shape, n_codes, bits):
    """Uniformly random packed code rows (unused high bits of the last word zero)."""
    W = -(-n_codes * bits // 32)
    w = g.integers(0, 1 << 32, size=shape + (W,), dtype=np.uint64).astype(np.uint32)
    spare = W * 32 - n_codes * bits
    if spare:
        w[..., -1] &= np.uint32((1 << (32 - spare)) - 1)
    return w


@pytest.mark.parametrize("method,bits", [("tq_prod", 3), ("tq_mse", 3), ("rq", 3), ("tq_prod", 4)])
def test_scores_many_tiles_per_cta(method, bits):
    """160 KV heads x 8,000 tokens: each CTA walks about 21 tiles, so both decode warpgroups
    cycle their code-stage rings and accumulators several times. Any code pattern is a valid
    key, so the keys are seeded random codes, norms and gammas; three heads are checked
    against the oracle's direct scores of the same codes."""
    n_heads, n_tok, group = 160, 8000, 8
    cb_bits = bits - 1 if method == "tq_prod" else bits
    c64 = codebook.lloyd_max(D, cb_bits)[0].astype(np.float32).astype(np.float64)
    c = torch.from_numpy(c64.astype(np.float32)).cuda()
    rot = torch.from_numpy(params.rotors(D, 1).astype(np.float32)).cuda()
    pi = torch.from_numpy(params.rotation(D, 2)).to(torch.float16).cuda()
    T = torch.from_numpy(params.qjl_matrix(D, D, 3)).to(torch.float16).cuda()
    g = np.random.default_rng(11)
    words = _random_words(g, (n_heads, n_tok), 129 if method == "rq" else D, cb_bits)
    nrm = np.exp(0.5 * g.standard_normal((n_heads, n_tok))).astype(np.float32).astype(np.float64)
    kw = {}
    if method == "rq":
        kw["rotors"] = rot
    else:
        kw["pi"] = pi
    if method == "tq_prod":
        swords = _random_words(g, (n_heads, n_tok), D, 1)
        gam = (0.3 * g.random((n_heads, n_tok))).astype(np.float32).astype(np.float64)
        kw.update(T=T, signs=_dev_words(swords), gammas=torch.from_numpy(gam.astype(np.float32)).cuda())
    q = torch.randn((n_heads, group, D), generator=torch.Generator().manual_seed(5)).to(torch.float16)
    mth = {"rq": kvrq.RQ_MSE, "tq_mse": kvrq.TQ_MSE, "tq_prod": kvrq.TQ_PROD}[method]
    s = kvrq.kv_score_packed(mth, q.cuda(), _dev_words(words), torch.from_numpy(nrm.astype(np.float32)).cuda(), bits,
                             n_tok, c, **kw)
    torch.cuda.synchronize()
    kvrq.device_status()
    p = {"centroids": c64, "rotors": rot.double().cpu().numpy(), "Pi": pi.double().cpu().numpy(),
         "T": T.double().cpu().numpy()}
    qf = q.double().numpy()
    for h in (0, 77, 159):
        kh = {"words": words[h:h + 1], "norms": nrm[h:h + 1]}
        if method == "tq_prod":
            kh["signs_words"] = swords[h:h + 1]
            kh["gammas"] = gam[h:h + 1]
        ref = score.direct(method, qf[h], kh, p, bits)
        compare_scores(s[h].double().cpu().numpy(), ref, score_tolerance(method, qf[h], kh, p, bits),
                       name="head %d" % h)
