"""Attention scores <q, k_hat> straight from packed keys, and by reconstruction.

* "TurboQuant 论文解读", "随机旋转（Lemma 1）": instead of turning every stored
  key back with Pi^T, rotate the query once (q' = Pi q) and take its inner
  product with the quantized rotated key.
* "TurboQuant + RotorQuant", "How TurboQuant Works":
  <q, k> ~ <q, k_mse> + ||r|| * sqrt(pi/2) / m * <S q, sign(S r)>.
* For RotorQuant the same identity holds group by group: <q, x_hat> =
  ||x|| * sum_g <R_g q_g R_g~, c_hat_g>, q zero-padded to 3G.
* "TurboQuant + RotorQuant", closing note of "When to Use Which": speed parity
  needs Q K^T computed directly from the compressed indices.

Grouped-query attention: query head h reads KV head h // (Hq / Hkv).
"""

import numpy as np

from . import codes as codes_mod, rq, tq
from .params import n_groups


def _kv_of(hq, n_q_heads, n_kv_heads):
    return hq // (n_q_heads // n_kv_heads)


def direct(method, q, keys, params, bits):
    """Scores [Hq, T] from packed keys, without reconstructing them.

    method: 'rq', 'tq_mse' or 'tq_prod'. q: [Hq, d]. keys: dict with
    'words' [Hkv, T, W], 'norms' [Hkv, T] and, for tq_prod, 'signs_words'
    [Hkv, T, m/32] and 'gammas' [Hkv, T]. params: dict with 'rotors' (rq) or
    'Pi' (and 'T' for tq_prod), and 'centroids' for the stored codes."""
    q = np.asarray(q, dtype=np.float64)
    Hq, d = q.shape
    words = np.asarray(keys["words"])
    Hkv, n_tok = words.shape[0], words.shape[1]
    c = np.asarray(params["centroids"], dtype=np.float64)
    out = np.zeros((Hq, n_tok))
    for h in range(Hq):
        kv = _kv_of(h, Hq, Hkv)
        norms = np.asarray(keys["norms"], dtype=np.float64)[kv]
        if method == "rq":
            G = n_groups(d)
            qp = rq.rotate(q[h : h + 1], params["rotors"])[0]  # rotated, padded query
            c_hat = c[codes_mod.unpack(words[kv], 3 * G, bits)]
            out[h] = norms * (c_hat @ qp)
        else:
            Pi = np.asarray(params["Pi"], dtype=np.float64)
            qp = Pi @ q[h]
            b_mse = bits if method == "tq_mse" else bits - 1
            c_hat = c[codes_mod.unpack(words[kv], d, b_mse)]
            s_mse = c_hat @ qp
            if method == "tq_prod":
                T = np.asarray(params["T"], dtype=np.float64)
                m = T.shape[0]
                s = 2 * codes_mod.unpack(np.asarray(keys["signs_words"])[kv], m, 1) - 1
                g = np.asarray(keys["gammas"], dtype=np.float64)[kv]
                s_mse = s_mse + (tq.QJL_SCALE_NUM / m) * g * (s @ (T @ qp))
            out[h] = norms * s_mse
    return out


def reconstruct(method, q, keys, params, bits):
    """Scores [Hq, T] by dequantizing every key and taking <q, k_hat>."""
    q = np.asarray(q, dtype=np.float64)
    Hq, d = q.shape
    words = np.asarray(keys["words"])
    Hkv = words.shape[0]
    out = []
    for h in range(Hq):
        kv = _kv_of(h, Hq, Hkv)
        norms = np.asarray(keys["norms"])[kv]
        if method == "rq":
            xh = rq.dequantize(words[kv], norms, params["rotors"], params["centroids"], bits, d)
        elif method == "tq_mse":
            xh = tq.mse_dequantize(words[kv], norms, params["Pi"], params["centroids"], bits, d)
        else:
            xh = tq.prod_dequantize(words[kv], np.asarray(keys["signs_words"])[kv], np.asarray(keys["gammas"])[kv],
                                    norms, params["Pi"], params["T"], params["centroids"], bits, d)
        out.append(xh @ q[h])
    return np.stack(out)
