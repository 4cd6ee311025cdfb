"""Full-size runs of the workloads the bench measures, checked on sampled rows against the oracle:
the Llama-3.1-8B-shaped KV stack (TurboQuant-prod keys, RotorQuant values), the Qwen2.5-3B decode
step (append + scores over 131,073 cached tokens) and the 1 GiB dimension sweep (d = 256, 1536, 4096)."""

import functools

import numpy as np
import pytest
import torch

import kv_cache_vector_rq_b200 as kvrq
from kv_cache_vector_rq_b200 import synth
from oracle import attention, codebook, codes as ocodes, params, rq, score, tq
from tests.parity import (attention_tolerance, compare_codes, compare_floats, compare_scores, compare_sketch_signs,
                          device_words, oracle_prod_inputs, random_words, score_tolerance, to_f64, words_u32)

pytestmark = pytest.mark.gpu

D = 128


@functools.lru_cache(maxsize=None)
def _pi64(d):
    return params.rotation(d, 2)


@functools.lru_cache(maxsize=None)
def _c(d, bits):
    return codebook.lloyd_max(d, bits)[0].astype(np.float32)


def _rows(n, k, seed):
    r = np.random.default_rng(seed).choice(n, k, replace=False)
    return np.unique(np.concatenate([r, [0, n - 1]]))


def _normwise(gpu, ref, rtol, skip=None):
    g, r = np.asarray(gpu, np.float64), np.asarray(ref, np.float64)
    keep = np.ones(len(g), bool) if skip is None else ~skip
    rn = np.linalg.norm(r[keep], axis=1)
    err = np.linalg.norm(g[keep] - r[keep], axis=1)
    ok = rn > 0
    assert np.all(err[ok] <= rtol * rn[ok]), "normwise relative error %g" % (err[ok] / rn[ok]).max()


def _check_prod(x_rows64, codes, signs, gammas, norms, pi64, T64, c64, bits, d):
    ref = tq.prod_quantize(x_rows64, pi64, T64, c64, bits)
    nb, bad = compare_codes(codes, ref, d, bits - 1, c64)
    assert np.allclose(norms, ref["norms"], rtol=1e-5)
    assert np.allclose(gammas[~bad], ref["gammas"][~bad], rtol=1e-4, atol=1e-7)
    compare_sketch_signs(signs, ref, x_rows64, pi64, T64, c64, skip_rows=bad)
    return bad, ref


def _plant_prod(ref, idx, codes, signs, gammas, norms):
    """Writes the oracle's codes of the sampled rows into the full-size device buffers (rows idx), so that
    the full-size launch that follows reads oracle-made inputs there; returns the float64 values of the
    fp32-rounded gammas and norms it wrote."""
    (oc, osg, og, on), g64, n64 = oracle_prod_inputs(ref)
    codes[idx], signs[idx], gammas[idx], norms[idx] = oc, osg, og, on
    return g64, n64


def test_config3_llama_kv_stack_sampled():
    """32 layers x 8 KV heads x 32,768 tokens x d=128 bf16: keys (rank-16 factor model + outliers)
    through TurboQuant-prod 3-bit, values N(0,1) through the RotorQuant 3-bit roundtrip."""
    layers, heads, tokens = 32, 8, 32768
    n = layers * heads * tokens
    k = synth.factor_keys(layers, heads, tokens, D, seed=21, dtype=torch.bfloat16, device="cuda").view(n, D)
    v = synth.gaussian(n, D, seed=22, dtype=torch.bfloat16, device="cuda")
    pi = torch.from_numpy(_pi64(D)).to(torch.bfloat16).cuda()
    T = torch.from_numpy(params.qjl_matrix(D, D, 3)).to(torch.float16).cuda()
    rot = torch.from_numpy(params.rotors(D, 1).astype(np.float32)).cuda()
    ck, cv = _c(D, 2), _c(D, 3)
    kc, ks, kg, kn = kvrq.tq_quantize_prod(k, pi, T, torch.from_numpy(ck).cuda(), 3)
    vc, vn, vh = kvrq.rq_quantize_dequantize(v, rot, torch.from_numpy(cv).cuda(), 3)
    torch.cuda.synchronize()
    kvrq.device_status()
    rows = _rows(n, 2048, 1)
    idx = torch.as_tensor(rows, device="cuda")
    pi64, T64 = to_f64(pi), to_f64(T)
    k64 = to_f64(k[idx])
    bad, ref = _check_prod(k64, words_u32(kc[idx]), words_u32(ks[idx]), to_f64(kg[idx]), to_f64(kn[idx]), pi64,
                           T64, ck.astype(np.float64), 3, D)
    # full-size dequantize with the oracle's codes planted at the sampled rows
    g64, n64 = _plant_prod(ref, idx, kc, ks, kg, kn)
    kh = kvrq.tq_dequantize(kc, kn, D, pi, torch.from_numpy(ck).cuda(), 3, signs=ks, gammas=kg, T=T)
    torch.cuda.synchronize()
    kvrq.device_status()
    xref = tq.prod_dequantize(ref["words"], ref["signs_words"], g64, n64, pi64, T64, ck.astype(np.float64), 3, D)
    _normwise(to_f64(kh[idx]), xref, 1e-2)
    v64 = to_f64(v[idx])
    rot64 = rot.double().cpu().numpy()
    ref = rq.roundtrip(v64, rot64, cv.astype(np.float64), 3)
    nb, badv = compare_codes(words_u32(vc[idx]), ref, 129, 3, cv.astype(np.float64))
    assert np.allclose(to_f64(vn[idx]), ref["norms"], rtol=1e-5)
    compare_floats(to_f64(vh[idx]), ref["xhat"], torch.bfloat16, ref["norms"], skip_rows=badv)


def test_config4_qwen_decode_step_sampled():
    """36 layers x 2 KV heads x (131,072 cached + 1 new) tokens, batch 1, 8 query heads per KV head:
    one append of a TurboQuant-prod key and a RotorQuant value per (layer, KV head), then scores of
    all 16 query heads over every token straight from the packed keys, and decode attention over the
    same cache. The appended slot is checked against the oracle's quantization of the new key and
    value; at 2,048 sampled slots of three heads the oracle's own codes of the same inputs are then
    planted and the full-size scores there are checked against the oracle; every token of two heads is
    then planted with seeded random codes and the full-size attention launch is checked element-wise
    against the oracle's attention over all of their tokens."""
    heads, cached, group, bits = 36 * 2, 131072, 8, 3
    t_max = cached + 1
    pi = torch.from_numpy(_pi64(D)).to(torch.float16).cuda()
    T = torch.from_numpy(params.qjl_matrix(D, D, 3)).to(torch.float16).cuda()
    rot = torch.from_numpy(params.rotors(D, 1).astype(np.float32)).cuda()
    ck, cv = _c(D, 2), _c(D, 3)
    ck_d, cv_d = torch.from_numpy(ck).cuda(), torch.from_numpy(cv).cuda()
    pi64, T64, rot64 = to_f64(pi), to_f64(T), rot.double().cpu().numpy()
    ck64, cv64 = ck.astype(np.float64), cv.astype(np.float64)
    Wk, Wv = kvrq.packed_words(D, 2), kvrq.packed_words(129, 3)
    k_codes = torch.empty((heads, t_max, Wk), dtype=torch.int32, device="cuda")
    k_signs = torch.empty((heads, t_max, D // 32), dtype=torch.int32, device="cuda")
    k_norms = torch.empty((heads, t_max), dtype=torch.float32, device="cuda")
    k_gam = torch.empty((heads, t_max), dtype=torch.float32, device="cuda")
    v_codes = torch.empty((heads, t_max, Wv), dtype=torch.int32, device="cuda")
    v_norms = torch.empty((heads, t_max), dtype=torch.float32, device="cuda")
    checked = (0, 35, 71)
    toks = _rows(t_max, 2048, 2)  # includes slot 0 and the appended slot `cached`
    tt = torch.as_tensor(toks, device="cuda")
    xk, xv = {}, {}  # inputs at the sampled slots of the checked heads
    for h0 in range(0, heads, 8):  # prefill every slot (the append then overwrites slot `cached`)
        h1 = min(heads, h0 + 8)
        r = (h1 - h0) * t_max
        kx = synth.lognormal(r, D, seed=50 + h0, dtype=torch.float16, device="cuda")
        vx = synth.gaussian(r, D, seed=60 + h0, dtype=torch.float16, device="cuda")
        kvrq.tq_quantize_prod(kx, pi, T, ck_d, bits, codes=k_codes[h0:h1].view(r, Wk), norms=k_norms[h0:h1].view(r),
                              signs=k_signs[h0:h1].view(r, D // 32), gammas=k_gam[h0:h1].view(r))
        kvrq.rq_quantize(vx, rot, cv_d, bits, codes=v_codes[h0:h1].view(r, Wv), norms=v_norms[h0:h1].view(r))
        for h in checked:
            if h0 <= h < h1:
                xk[h] = to_f64(kx.view(h1 - h0, t_max, D)[h - h0, tt])
                xv[h] = to_f64(vx.view(h1 - h0, t_max, D)[h - h0, tt])
        del kx, vx
    new_k = synth.lognormal(heads, D, seed=10, dtype=torch.float16, device="cuda")
    new_v = synth.gaussian(heads, D, seed=11, dtype=torch.float16, device="cuda")
    q = synth.gaussian(heads * group, D, seed=9, dtype=torch.float16, device="cuda").view(heads, group, D)
    kvrq.kv_cache_append(kvrq.TQ_PROD, new_k, cached, bits, ck_d, k_codes, k_norms, pi=pi, T=T, signs=k_signs,
                         gammas=k_gam)
    kvrq.kv_cache_append(kvrq.RQ_MSE, new_v, cached, bits, cv_d, v_codes, v_norms, rotors=rot)
    torch.cuda.synchronize()
    kvrq.device_status()
    # the appended slot holds the quantization of the new key and value
    _check_prod(to_f64(new_k), words_u32(k_codes[:, cached]), words_u32(k_signs[:, cached]),
                to_f64(k_gam[:, cached]), to_f64(k_norms[:, cached]), pi64, T64, ck64, bits, D)
    refv = rq.quantize(to_f64(new_v), rot64, cv64, bits)
    compare_codes(words_u32(v_codes[:, cached]), refv, 129, bits, cv64)
    # plant the oracle's codes of the sampled slots' inputs (the appended slot: the new key and value)
    planted = {}
    for h in checked:
        xk[h][-1], xv[h][-1] = to_f64(new_k[h]), to_f64(new_v[h])
        refk = tq.prod_quantize(xk[h], pi64, T64, ck64, bits)
        g64, n64 = _plant_prod(refk, (h, tt), k_codes, k_signs, k_gam, k_norms)
        rv = rq.quantize(xv[h], rot64, cv64, bits)
        vn32 = rv["norms"].astype(np.float32)
        v_codes[h, tt] = device_words(rv["words"])
        v_norms[h, tt] = torch.from_numpy(vn32).cuda()
        planted[h] = ({"words": refk["words"][None], "norms": n64[None], "signs_words": refk["signs_words"][None],
                       "gammas": g64[None]}, {"words": rv["words"][None], "norms": vn32.astype(np.float64)[None]})
    s = kvrq.kv_score_packed(kvrq.TQ_PROD, q, k_codes, k_norms, bits, t_max, ck_d, pi=pi, T=T, signs=k_signs,
                             gammas=k_gam)
    torch.cuda.synchronize()
    kvrq.device_status()
    p = {"centroids": ck64, "Pi": pi64, "T": T64}
    qf = q.double().cpu().numpy()
    for h in checked:
        kh = planted[h][0]
        ref = score.direct("tq_prod", qf[h], kh, p, bits)
        compare_scores(s[h][:, toks].double().cpu().numpy(), ref, score_tolerance("tq_prod", qf[h], kh, p, bits),
                       name="head %d" % h)
    del s
    # decode attention over the full cache: every token of two heads is planted with seeded random codes, norms
    # and gammas (any code row is a valid key or value), and the full-size launch is compared element-wise with
    # the oracle's attention over all 131,073 tokens of those heads
    g = np.random.default_rng(4)
    full_heads = (0, heads - 1)
    cache = {}
    for h in full_heads:
        kh = {"words": random_words(g, (1, t_max), D, 2), "signs_words": random_words(g, (1, t_max), D, 1),
              "norms": np.exp(0.5 * g.standard_normal((1, t_max))).astype(np.float32).astype(np.float64),
              "gammas": (0.3 * g.random((1, t_max))).astype(np.float32).astype(np.float64)}
        vh = {"words": random_words(g, (1, t_max), 129, 3),
              "norms": np.exp(0.5 * g.standard_normal((1, t_max))).astype(np.float32).astype(np.float64)}
        k_codes[h] = device_words(kh["words"][0])
        k_signs[h] = device_words(kh["signs_words"][0])
        k_norms[h] = torch.from_numpy(kh["norms"][0].astype(np.float32)).cuda()
        k_gam[h] = torch.from_numpy(kh["gammas"][0].astype(np.float32)).cuda()
        v_codes[h] = device_words(vh["words"][0])
        v_norms[h] = torch.from_numpy(vh["norms"][0].astype(np.float32)).cuda()
        cache[h] = (kh, vh)
    full = kvrq.kv_attention_packed(kvrq.TQ_PROD, q, k_codes, k_norms, bits, v_codes, v_norms, bits, t_max, ck_d,
                                    rot, cv_d, pi=pi, T=T, k_signs=k_signs, k_gammas=k_gam)
    torch.cuda.synchronize()
    kvrq.device_status()
    assert torch.isfinite(full).all()
    rel = 1e-2 if kvrq.attention_uses_tensor_cores(kvrq.TQ_PROD, bits, bits, group) else 1e-3
    vp = {"rotors": rot64, "centroids": cv64}
    for h in full_heads:
        kh, vh = cache[h]
        ref = attention.decode("tq_prod", qf[h], kh, p, bits, vh, vp, bits, 1.0 / np.sqrt(D))
        vmax = np.abs(attention.values_hat(vh, vp, bits, D)).max()
        err = np.abs(full[h].double().cpu().numpy() - ref)
        tol = attention_tolerance(ref, vmax, rel)
        assert np.all(err <= tol), "attention head %d: max excess %g" % (h, float((err - tol).max()))
    # every full-size output is a convex combination of value reconstructions: bounded by the largest one
    vbound = float(v_norms.max()) * float(np.abs(cv64).max()) * np.sqrt(3.0) * 1.001
    assert float(full.abs().max()) <= vbound


@pytest.mark.parametrize("d", [256, 1536, 4096])
def test_config5_dimension_sweep_sampled(d):
    """1 GiB of fp16 rows (N(0,1) directions, LogNormal(0, 0.5) norms) at d: the RotorQuant 3-bit
    roundtrip and the TurboQuant-prod 3-bit quantize + dequantize (m = d), sampled rows vs the oracle."""
    n = (1 << 30) // (2 * d)
    x = synth.lognormal(n, d, seed=5 + d, dtype=torch.float16, device="cuda", outliers=())
    rot = torch.from_numpy(params.rotors(d, 1).astype(np.float32)).cuda()
    c3 = _c(d, 3)
    codes, norms, xhat = kvrq.rq_quantize_dequantize(x, rot, torch.from_numpy(c3).cuda(), 3)
    torch.cuda.synchronize()
    kvrq.device_status()
    rows = _rows(n, 256, 3)
    idx = torch.as_tensor(rows, device="cuda")
    ref = rq.roundtrip(to_f64(x[idx]), rot.double().cpu().numpy(), c3.astype(np.float64), 3)
    G = kvrq.rq_groups(d)
    nb, bad = compare_codes(words_u32(codes[idx]), ref, 3 * G, 3, c3.astype(np.float64))
    assert np.allclose(to_f64(norms[idx]), ref["norms"], rtol=1e-5)
    compare_floats(to_f64(xhat[idx]), ref["xhat"], torch.float16, ref["norms"], skip_rows=bad)
    del codes, norms, xhat
    pi = torch.from_numpy(_pi64(d)).to(torch.float16).cuda()
    T = torch.from_numpy(params.qjl_matrix(d, d, 3)).to(torch.float16).cuda()
    c2 = _c(d, 2)
    kc, ks, kg, kn = kvrq.tq_quantize_prod(x, pi, T, torch.from_numpy(c2).cuda(), 3)
    torch.cuda.synchronize()
    kvrq.device_status()
    rows = _rows(n, 128, 4)
    idx = torch.as_tensor(rows, device="cuda")
    pi64, T64 = to_f64(pi), to_f64(T)
    bad, ref = _check_prod(to_f64(x[idx]), words_u32(kc[idx]), words_u32(ks[idx]), to_f64(kg[idx]), to_f64(kn[idx]),
                           pi64, T64, c2.astype(np.float64), 3, d)
    # full-size dequantize with the oracle's codes planted at the sampled rows
    g64, n64 = _plant_prod(ref, idx, kc, ks, kg, kn)
    kh = kvrq.tq_dequantize(kc, kn, d, pi, torch.from_numpy(c2).cuda(), 3, signs=ks, gammas=kg, T=T)
    torch.cuda.synchronize()
    kvrq.device_status()
    xref = tq.prod_dequantize(ref["words"], ref["signs_words"], g64, n64, pi64, T64, c2.astype(np.float64), 3, d)
    _normwise(to_f64(kh[idx]), xref, 2e-3)
