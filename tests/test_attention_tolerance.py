"""The decode-attention parity rule on the CPU: a float32 restatement of the kernels' algorithm
(logits from rotated queries, online softmax over 256-token chunks, value sums in the rotated
domain, one inverse sandwich after the merge) passes it, and each plausible kernel mistake,
planted in that restatement, fails it. A restatement with the operands of a tensor-core version
(fp16 rotated queries, T q', centroids and weights, fp32 sums, 128-token tiles) stays inside the
1e-2 bound of the tensor-core paths."""

import numpy as np
import pytest

from oracle import attention, codebook, codes as ocodes, params, rq, tq
from tests.parity import attention_tolerance

D = 128
F = np.float32


def _cache(n_kv, n_tok, seed):
    g = np.random.default_rng(seed)
    kp = {"centroids": codebook.lloyd_max(D, 2)[0].astype(F).astype(np.float64),
          "Pi": params.rotation(D, 2).astype(np.float16).astype(np.float64),
          "T": params.qjl_matrix(D, D, 3).astype(np.float16).astype(np.float64)}
    vp = {"centroids": codebook.lloyd_max(D, 3)[0].astype(F).astype(np.float64),
          "rotors": params.rotors(D, 4).astype(F).astype(np.float64)}
    keys = {"words": [], "norms": [], "signs_words": [], "gammas": []}
    values = {"words": [], "norms": []}
    for h in range(n_kv):
        k = g.standard_normal((n_tok, D)) * np.exp(0.5 * g.standard_normal((n_tok, 1)))
        qq = tq.prod_quantize(k, kp["Pi"], kp["T"], kp["centroids"], 3)
        for key in ("words", "signs_words"):
            keys[key].append(qq[key])
        keys["norms"].append(qq["norms"].astype(F).astype(np.float64))
        keys["gammas"].append(qq["gammas"].astype(F).astype(np.float64))
        vq = rq.quantize(g.standard_normal((n_tok, D)), vp["rotors"], vp["centroids"], 3)
        values["words"].append(vq["words"])
        values["norms"].append(vq["norms"].astype(F).astype(np.float64))
    return ({kk: np.stack(v) for kk, v in keys.items()}, kp, {kk: np.stack(v) for kk, v in values.items()}, vp)


def _f32_kernel(q, keys, kp, values, vp, scale, chunk=256, mistake=None):
    """TurboQuant-prod 3-bit keys, RotorQuant 3-bit values, the kernels' order of work in float32."""
    Hq, Hkv = q.shape[0], keys["words"].shape[0]
    group = Hq // Hkv
    n_tok = keys["words"].shape[1]
    qjl = F(np.sqrt(np.pi / 2) / D)
    out = np.zeros((Hq, D), dtype=F)
    for h in range(Hq):
        kv = (h % Hkv) if mistake == "gqa" else h // group
        qp = (kp["Pi"].astype(F) @ q[h].astype(F)).astype(F)
        sq = (kp["T"].astype(F) @ qp).astype(F)
        c = kp["centroids"].astype(F)[ocodes.unpack(keys["words"][kv], D, 2)]
        s = (2 * ocodes.unpack(keys["signs_words"][kv], D, 1) - 1).astype(F)
        dot = c @ qp
        if mistake != "no_qjl":
            dot = dot + qjl * keys["gammas"][kv].astype(F) * (s @ sq)
        lg = (F(1.0 if mistake == "no_scale" else scale) * keys["norms"][kv].astype(F) * dot).astype(F)
        cv = vp["centroids"].astype(F)[ocodes.unpack(values["words"][kv], 129, 3)]
        vn = values["norms"][kv].astype(F)
        if mistake == "no_vnorm":
            vn = np.ones_like(vn)
        ms, ls, accs = [], [], []
        for t0 in range(0, n_tok, chunk):
            l_c = lg[t0:t0 + chunk]
            m = l_c.max()
            w = np.exp(l_c - m).astype(F)
            ms.append(m)
            ls.append(w.sum(dtype=F))
            accs.append(((w * vn[t0:t0 + chunk]) @ cv[t0:t0 + chunk]).astype(F))
        ms, ls, accs = np.array(ms, F), np.array(ls, F), np.array(accs, F)
        if mistake == "no_rescale":  # chunks merged without bringing them to a common max
            y = accs.sum(axis=0) / ls.sum()
        else:
            wc = np.exp(ms - ms.max()).astype(F)
            y = (wc @ accs) / (wc @ ls)
        if mistake == "no_unrotate":
            out[h] = y[:D]
        else:
            out[h] = rq.unrotate(y[None].astype(np.float64), vp["rotors"], D)[0].astype(F)
    return out


@pytest.fixture(scope="module")
def case():
    keys, kp, values, vp = _cache(2, 700, seed=1)  # three chunks of 256, the last ragged
    q = np.random.default_rng(2).standard_normal((8, D)).astype(np.float16).astype(np.float64) * 2
    scale = 1.0 / np.sqrt(D)
    ref = attention.decode("tq_prod", q, keys, kp, 3, values, vp, 3, scale)
    vmax = max(np.abs(attention.values_hat({kk: v[h:h + 1] for kk, v in values.items()}, vp, 3, D)).max()
               for h in range(2))
    return q, keys, kp, values, vp, scale, ref, attention_tolerance(ref, vmax)


def test_float32_restatement_passes(case):
    q, keys, kp, values, vp, scale, ref, tol = case
    got = _f32_kernel(q, keys, kp, values, vp, scale)
    assert np.all(np.abs(got - ref) <= tol)
    assert np.abs(got - ref).max() < 0.05 * tol.min()  # far inside the bound


@pytest.mark.parametrize("mistake", ["gqa", "no_qjl", "no_scale", "no_vnorm", "no_rescale", "no_unrotate"])
def test_planted_kernel_mistake_fails(case, mistake):
    q, keys, kp, values, vp, scale, ref, tol = case
    got = _f32_kernel(q, keys, kp, values, vp, scale, mistake=mistake)
    assert np.any(np.abs(got - ref) > tol), mistake


def _fp16_operands(q, keys, kp, values, vp, scale, tile=128):
    """The same algorithm with fp16 operands for both contractions (fp32 sums); the rotated pad
    coordinate stays in fp32, as it would on the CUDA cores."""
    H = np.float16
    Hq, Hkv = q.shape[0], keys["words"].shape[0]
    group = Hq // Hkv
    n_tok = keys["words"].shape[1]
    qjl = F(np.sqrt(np.pi / 2) / D)
    out = np.zeros((Hq, D))
    for h in range(Hq):
        kv = h // group
        qp = (kp["Pi"] @ q[h]).astype(F)
        sq = (kp["T"] @ qp.astype(np.float64)).astype(F)
        c = kp["centroids"][ocodes.unpack(keys["words"][kv], D, 2)].astype(H).astype(F)
        s = (2 * ocodes.unpack(keys["signs_words"][kv], D, 1) - 1).astype(F)
        dot = c @ qp.astype(H).astype(F) + qjl * keys["gammas"][kv].astype(F) * (s @ sq.astype(H).astype(F))
        lg = (F(scale) * keys["norms"][kv].astype(F) * dot).astype(F)
        cv = vp["centroids"][ocodes.unpack(values["words"][kv], 129, 3)].astype(F)
        vn = values["norms"][kv].astype(F)
        m, l, acc = -np.inf, F(0), np.zeros(129, F)
        for t0 in range(0, n_tok, tile):
            lt = lg[t0:t0 + tile]
            mn = max(m, lt.max())
            al = np.exp(F(m - mn)) if np.isfinite(m) else F(0)
            p = np.exp(lt - mn).astype(F)
            l = l * al + p.sum(dtype=F)
            pw = (p * vn[t0:t0 + tile]).astype(F)
            acc = acc * al
            acc[:128] += pw.astype(H).astype(F) @ cv[t0:t0 + tile, :128].astype(H).astype(F)
            acc[128] += pw @ cv[t0:t0 + tile, 128]
            m = mn
        out[h] = rq.unrotate((acc / l)[None].astype(np.float64), vp["rotors"], D)[0]
    return out


def test_fp16_operand_restatement_within_tensor_core_bound():
    keys, kp, values, vp = _cache(2, 2000, seed=5)
    q = np.random.default_rng(6).standard_normal((8, D)).astype(np.float16).astype(np.float64) * 2
    scale = 1.0 / np.sqrt(D)
    ref = attention.decode("tq_prod", q, keys, kp, 3, values, vp, 3, scale)
    vmax = max(np.abs(attention.values_hat({kk: v[h:h + 1] for kk, v in values.items()}, vp, 3, D)).max()
               for h in range(2))
    got = _fp16_operands(q, keys, kp, values, vp, scale)
    err = np.abs(got - ref)
    assert np.all(err <= attention_tolerance(ref, vmax, rel=1e-2))
    assert (err / np.abs(ref).max(axis=1, keepdims=True)).max() < 5e-3
