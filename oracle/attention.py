"""Decode attention over a packed KV cache: softmax(q K_hat^T * scale) V_hat.

TEST INFRASTRUCTURE ONLY (see the package docstring).

* "TurboQuant и PolarQuant: математика квантизации KV-кэша в LLM", section
  "Проблема KV-кэша в трансформерах": attention weights are the softmax of the
  query's dot products with every key over sqrt(d), and the output is the
  weighted sum of the values.
* "TurboQuant + RotorQuant", closing note of "When to Use Which": speed parity
  needs attention computed from the compressed indices instead of
  decompressing the cache first.

The oracle takes the plain definition: every key and every value is
dequantized (keys by any of the three quantizers, values by RotorQuant), the
logits are scale * <q, k_hat_t>, the weights their softmax over the tokens
(evaluated with the largest logit subtracted, which leaves the quotient
unchanged), and the output the weighted sum of the v_hat_t.

Grouped-query attention: query head h reads KV head h // (Hq / Hkv).
"""

import numpy as np

from . import rq, score


def softmax(s):
    """Softmax over the last axis of a float64 array."""
    s = np.asarray(s, dtype=np.float64)
    e = np.exp(s - s.max(axis=-1, keepdims=True))
    return e / e.sum(axis=-1, keepdims=True)


def values_hat(values, v_params, v_bits, d):
    """RotorQuant-dequantized values [Hkv, T, d] of the packed value cache."""
    words = np.asarray(values["words"])
    norms = np.asarray(values["norms"], dtype=np.float64)
    return np.stack([rq.dequantize(words[h], norms[h], v_params["rotors"], v_params["centroids"], v_bits, d)
                     for h in range(words.shape[0])])


def decode(k_method, q, keys, k_params, k_bits, values, v_params, v_bits, scale):
    """Attention outputs [Hq, d] for one decode step.

    q: [Hq, d]. keys / k_params / k_bits: as for score.reconstruct (method 'rq',
    'tq_mse' or 'tq_prod'). values: dict with 'words' [Hkv, T, Wv] and 'norms'
    [Hkv, T] of RotorQuant codes; v_params: 'rotors' and 'centroids' of the
    value quantizer. scale multiplies the logits (1/sqrt(d) in the pages)."""
    q = np.asarray(q, dtype=np.float64)
    Hq, d = q.shape
    logits = scale * score.reconstruct(k_method, q, keys, k_params, k_bits)  # [Hq, T]
    w = softmax(logits)
    v_hat = values_hat(values, v_params, v_bits, d)  # [Hkv, T, d]
    Hkv = v_hat.shape[0]
    out = np.zeros((Hq, d))
    for h in range(Hq):
        out[h] = w[h] @ v_hat[h // (Hq // Hkv)]
    return out


def decode_paged(k_method, q, pool_keys, slots, k_params, k_bits, pool_values, v_params, v_bits, scale):
    """decode() over a paged pool: token t of KV head h is pool row slots[h][t] of every array in
    pool_keys / pool_values (each [pool_rows, ...]); the tokens are gathered in order, then
    attended by the plain definition."""
    keys = {kk: np.stack([np.asarray(v)[np.asarray(s)] for s in slots]) for kk, v in pool_keys.items()}
    values = {kk: np.stack([np.asarray(v)[np.asarray(s)] for s in slots]) for kk, v in pool_values.items()}
    return decode(k_method, q, keys, k_params, k_bits, values, v_params, v_bits, scale)
