"""Pins of the oracle's decode attention over a packed cache.

Each check fixes the result by something other than the oracle itself: the
softmax of one logit is 1, logits that are all equal give the mean, a dominant
logit picks its token, and on small cases the whole step equals PyTorch's own
scaled_dot_product_attention (float64, CPU) run on the oracle's dequantized
keys and values, with grouped-query heads expanded by repeat_interleave."""

import numpy as np
import pytest
import torch

from oracle import attention, codebook, params, rq, tq

D = 128


def _cache(k_method, k_bits, v_bits, n_kv, n_tok, seed):
    g = np.random.default_rng(seed)
    kb = k_bits - 1 if k_method == "tq_prod" else k_bits
    kp = {"centroids": codebook.lloyd_max(D, kb)[0], "rotors": params.rotors(D, 1), "Pi": params.rotation(D, 2),
          "T": params.qjl_matrix(D, D, 3)}
    vp = {"centroids": codebook.lloyd_max(D, v_bits)[0], "rotors": params.rotors(D, 4)}
    keys = {"words": [], "norms": [], "signs_words": [], "gammas": []}
    values = {"words": [], "norms": []}
    k_hat, v_hat = [], []
    for h in range(n_kv):
        k = g.standard_normal((n_tok, D)) * np.exp(0.5 * g.standard_normal((n_tok, 1)))
        v = g.standard_normal((n_tok, D))
        if k_method == "rq":
            qq = rq.quantize(k, kp["rotors"], kp["centroids"], k_bits)
            k_hat.append(rq.dequantize(qq["words"], qq["norms"], kp["rotors"], kp["centroids"], k_bits, D))
        elif k_method == "tq_mse":
            qq = tq.mse_quantize(k, kp["Pi"], kp["centroids"], k_bits)
            k_hat.append(tq.mse_dequantize(qq["words"], qq["norms"], kp["Pi"], kp["centroids"], k_bits, D))
        else:
            qq = tq.prod_quantize(k, kp["Pi"], kp["T"], kp["centroids"], k_bits)
            keys["signs_words"].append(qq["signs_words"])
            keys["gammas"].append(qq["gammas"])
            k_hat.append(tq.prod_dequantize(qq["words"], qq["signs_words"], qq["gammas"], qq["norms"], kp["Pi"],
                                            kp["T"], kp["centroids"], k_bits, D))
        keys["words"].append(qq["words"])
        keys["norms"].append(qq["norms"])
        vq = rq.quantize(v, vp["rotors"], vp["centroids"], v_bits)
        values["words"].append(vq["words"])
        values["norms"].append(vq["norms"])
        v_hat.append(rq.dequantize(vq["words"], vq["norms"], vp["rotors"], vp["centroids"], v_bits, D))
    keys = {kk: np.stack(v) for kk, v in keys.items() if v}
    values = {kk: np.stack(v) for kk, v in values.items()}
    return keys, kp, values, vp, np.stack(k_hat), np.stack(v_hat)


@pytest.mark.parametrize("k_method,k_bits", [("rq", 3), ("tq_mse", 2), ("tq_prod", 3)])
def test_equals_torch_sdpa_on_dequantized_cache(k_method, k_bits):
    n_kv, group, n_tok, v_bits = 2, 4, 37, 3
    keys, kp, values, vp, k_hat, v_hat = _cache(k_method, k_bits, v_bits, n_kv, n_tok, seed=k_bits)
    q = np.random.default_rng(9).standard_normal((n_kv * group, D))
    scale = 1.0 / np.sqrt(D)
    got = attention.decode(k_method, q, keys, kp, k_bits, values, vp, v_bits, scale)
    K = torch.from_numpy(k_hat).repeat_interleave(group, dim=0)  # [Hq, T, d]
    V = torch.from_numpy(v_hat).repeat_interleave(group, dim=0)
    Q = torch.from_numpy(q)[:, None, :]  # [Hq, 1, d]
    ref = torch.nn.functional.scaled_dot_product_attention(Q, K, V, scale=scale)[:, 0, :].numpy()
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


def test_one_token_returns_its_value():
    keys, kp, values, vp, _, v_hat = _cache("rq", 3, 2, 2, 1, seed=1)
    q = np.random.default_rng(2).standard_normal((4, D)) * 10.0
    got = attention.decode("rq", q, keys, kp, 3, values, vp, 2, 1.0)
    for h in range(4):
        np.testing.assert_allclose(got[h], v_hat[h // 2, 0], rtol=0, atol=1e-13)


def test_zero_scale_gives_the_mean_value():
    keys, kp, values, vp, _, v_hat = _cache("tq_prod", 3, 3, 1, 50, seed=3)
    q = np.random.default_rng(4).standard_normal((2, D))
    got = attention.decode("tq_prod", q, keys, kp, 3, values, vp, 3, 0.0)
    np.testing.assert_allclose(got, np.repeat(v_hat.mean(axis=1), 2, axis=0), rtol=0, atol=1e-13)


def test_dominant_logit_selects_its_token():
    keys, kp, values, vp, k_hat, v_hat = _cache("tq_mse", 3, 4, 1, 20, seed=5)
    q = np.random.default_rng(6).standard_normal((1, D))
    logits = k_hat[0] @ q[0]
    top = int(np.argmax(logits))
    gap = logits[top] - np.sort(logits)[-2]
    assert gap > 0
    got = attention.decode("tq_mse", q, keys, kp, 3, values, vp, 4, 60.0 / gap)  # others weigh < e^-60
    np.testing.assert_allclose(got[0], v_hat[0, top], rtol=0, atol=1e-12)


def test_softmax_shift_and_sum():
    s = np.random.default_rng(0).standard_normal((3, 11)) * 30
    p = attention.softmax(s)
    np.testing.assert_allclose(p.sum(axis=-1), 1.0, rtol=0, atol=1e-15)
    np.testing.assert_allclose(attention.softmax(s + 1234.5), p, rtol=1e-12, atol=0)
    np.testing.assert_allclose(p[0], np.exp(s[0]) / np.exp(s[0]).sum(), rtol=1e-12, atol=0)


def test_paged_pool_with_shuffled_pages_equals_the_contiguous_cache():
    import kv_cache_vector_rq_b200 as kvrq

    n_kv, group, n_tok, P = 2, 4, 45, 8
    keys, kp, values, vp, _, _ = _cache("tq_prod", 3, 3, n_kv, n_tok, seed=7)
    q = np.random.default_rng(8).standard_normal((n_kv * group, D))
    ref = attention.decode("tq_prod", q, keys, kp, 3, values, vp, 3, 0.1)
    # place each head's tokens through the page manager; interleave appends so pages alternate
    pc = kvrq.PagedCache(32, P)
    sids = [pc.add_seq() for _ in range(n_kv)]
    for t0 in range(0, n_tok, 5):
        for s in sids:
            pc.append(s, min(5, n_tok - t0))
    slots = [pc.slots(s, 0, n_tok) for s in sids]
    rows = 32 * P
    pool_k = {kk: np.zeros((rows,) + v.shape[2:], dtype=v.dtype) for kk, v in keys.items()}
    pool_v = {kk: np.zeros((rows,) + v.shape[2:], dtype=v.dtype) for kk, v in values.items()}
    for h in range(n_kv):
        for kk in keys:
            pool_k[kk][slots[h]] = keys[kk][h]
        for kk in values:
            pool_v[kk][slots[h]] = values[kk][h]
    assert len(set(np.concatenate(slots).tolist())) == n_kv * n_tok  # disjoint slots
    got = attention.decode_paged("tq_prod", q, pool_k, slots, kp, 3, pool_v, vp, 3, 0.1)
    np.testing.assert_array_equal(got, ref)
