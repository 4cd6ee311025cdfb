"""GPU parity of the paged-cache paths ("TurboQuant + RotorQuant", "Post-Prefill Quantization": a prefill cache
quantized in bulk, then one new key and value per decode step, the packed rows of many sequences in pages of a
pool): kv_score_packed_paged, kv_attention_packed_paged and kv_cache_append_rows, through the C ABI.

Pages are handed out by the library's page manager (kvrq.PagedCache) to sequences of different lengths whose
appends interleave, so a sequence's pages are scattered through the pool. Pools hold seeded random codes, norms
and gammas (any code row is a valid key or value). The oracle gathers each sequence's tokens by slot
(oracle/attention.py decode_paged; score.direct on the gathered keys)."""

import numpy as np
import pytest
import torch

import kv_cache_vector_rq_b200 as kvrq
from oracle import attention, codebook, codes as ocodes, params, rq, score, tq
from tests.parity import (attention_tolerance, compare_codes, compare_scores, compare_sketch_signs, device_words,
                          random_words, score_tolerance, to_f64, words_u32)

pytestmark = pytest.mark.gpu

D = 128


def _build_pages(page_tokens, lens, chunk, seed):
    """Sequences of lengths `lens` appended in turns of `chunk` tokens (interleaving their pages); returns the
    page manager, block tables [n_seqs, ld_table] int32, the slot list of every sequence and the pool size."""
    n_pages = sum(-(-L // page_tokens) for L in lens) + 3
    pc = kvrq.PagedCache(n_pages, page_tokens)
    seqs = [pc.add_seq() for _ in lens]
    done = [0] * len(lens)
    g = np.random.default_rng(seed)
    while any(done[i] < lens[i] for i in range(len(lens))):
        i = int(g.integers(len(lens)))
        k = min(chunk, lens[i] - done[i])
        if k > 0:
            pc.append(seqs[i], k)
            done[i] += k
    tables = [pc.block_table(s)[0] for s in seqs]
    ld = max(len(t) for t in tables)
    bt = np.zeros((len(lens), ld), dtype=np.int32)
    for i, t in enumerate(tables):
        bt[i, :len(t)] = t
    slots = [pc.slots(s, 0, L) for s, L in zip(seqs, lens)]
    return pc, bt, slots, n_pages * page_tokens


def _params(k_method, k_bits, v_bits=3):
    cb = k_bits - 1 if k_method == "tq_prod" else k_bits
    kc = codebook.lloyd_max(D, cb)[0].astype(np.float32).astype(np.float64)
    vc = codebook.lloyd_max(D, v_bits)[0].astype(np.float32).astype(np.float64)
    pi = torch.from_numpy(params.rotation(D, 2)).to(torch.float16)
    T = torch.from_numpy(params.qjl_matrix(D, D, 3)).to(torch.float16)
    kp = {"centroids": kc, "rotors": params.rotors(D, 1).astype(np.float32).astype(np.float64),
          "Pi": pi.double().numpy(), "T": T.double().numpy()}
    vp = {"centroids": vc, "rotors": params.rotors(D, 4).astype(np.float32).astype(np.float64)}
    return kp, vp, pi, T


def _pools(k_method, k_bits, v_bits, pool_heads, n_slots, seed):
    g = np.random.default_rng(seed)
    cb = k_bits - 1 if k_method == "tq_prod" else k_bits
    nck = 129 if k_method == "rq" else D
    pools = {"k_words": random_words(g, (pool_heads, n_slots), nck, cb),
             "k_norms": np.exp(0.5 * g.standard_normal((pool_heads, n_slots))).astype(np.float32),
             "v_words": random_words(g, (pool_heads, n_slots), 129, v_bits),
             "v_norms": np.exp(0.5 * g.standard_normal((pool_heads, n_slots))).astype(np.float32)}
    if k_method == "tq_prod":
        pools["k_signs"] = random_words(g, (pool_heads, n_slots), D, 1)
        pools["k_gammas"] = (0.3 * g.random((pool_heads, n_slots))).astype(np.float32)
    return pools


def _dev(a):
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint32:
        return device_words(a)
    return torch.from_numpy(a).cuda()


CASES = [("tq_prod", 3, 16, 8), ("tq_prod", 3, 128, 8), ("tq_prod", 3, 48, 8), ("rq", 3, 16, 16), ("tq_mse", 3, 32, 5)]


@pytest.mark.parametrize("k_method,k_bits,page_tokens,group", CASES)
def test_paged_scores_and_attention(k_method, k_bits, page_tokens, group):
    layers, kv_heads = 2, 2
    lens = [700, 1, 2100]
    n_seqs = len(lens)
    pc, bt, slots, n_slots = _build_pages(page_tokens, lens, chunk=37, seed=page_tokens)
    pool_heads = layers * kv_heads
    kp, vp, pi, T = _params(k_method, k_bits)
    pools = _pools(k_method, k_bits, 3, pool_heads, n_slots, seed=page_tokens + group)
    n_heads = layers * n_seqs * kv_heads
    q = (2.0 * torch.randn((n_heads, group, D), generator=torch.Generator().manual_seed(group))).to(torch.float16)
    method = {"rq": kvrq.RQ_MSE, "tq_mse": kvrq.TQ_MSE, "tq_prod": kvrq.TQ_PROD}[k_method]
    kw = dict(rotors=_dev(kp["rotors"].astype(np.float32))) if k_method == "rq" else dict(pi=pi.cuda())
    if k_method == "tq_prod":
        kw.update(T=T.cuda(), signs=_dev(pools["k_signs"]), gammas=_dev(pools["k_gammas"]))
    bt_d = torch.from_numpy(bt).cuda()
    sl_d = torch.tensor(lens, dtype=torch.int32, device="cuda")
    max_tokens = max(lens)
    sentinel = -7.0
    scores = torch.full((n_heads, group, max_tokens), sentinel, dtype=torch.float32, device="cuda")
    kvrq.kv_score_packed_paged(method, q.cuda(), _dev(pools["k_words"]), _dev(pools["k_norms"]), k_bits, bt_d, sl_d,
                               page_tokens, n_seqs, kv_heads, max_tokens,
                               _dev(kp["centroids"].astype(np.float32)), scores=scores, **kw)
    akw = dict(k_rotors=kw["rotors"]) if k_method == "rq" else dict(pi=kw["pi"])
    if k_method == "tq_prod":
        akw.update(T=kw["T"], k_signs=kw["signs"], k_gammas=kw["gammas"])
    assert kvrq.attention_uses_tensor_cores(method, k_bits, 3, group)
    out = kvrq.kv_attention_packed_paged(method, q.cuda(), _dev(pools["k_words"]), _dev(pools["k_norms"]), k_bits,
                                         _dev(pools["v_words"]), _dev(pools["v_norms"]), 3, bt_d, sl_d, page_tokens,
                                         n_seqs, kv_heads, max_tokens, _dev(kp["centroids"].astype(np.float32)),
                                         _dev(vp["rotors"].astype(np.float32)), _dev(vp["centroids"].astype(np.float32)),
                                         **akw)
    torch.cuda.synchronize()
    kvrq.device_status()
    got_s = scores.double().cpu().numpy()
    got_o = out.double().cpu().numpy()
    qf = q.double().numpy()
    pk = {"words": pools["k_words"], "norms": pools["k_norms"].astype(np.float64)}
    if k_method == "tq_prod":
        pk.update(signs_words=pools["k_signs"], gammas=pools["k_gammas"].astype(np.float64))
    pv = {"words": pools["v_words"], "norms": pools["v_norms"].astype(np.float64)}
    for h in range(n_heads):
        k = h % kv_heads
        s = (h // kv_heads) % n_seqs
        layer = h // (kv_heads * n_seqs)
        p = layer * kv_heads + k
        L = lens[s]
        kh = {kk: v[p][slots[s]][None] for kk, v in pk.items()}
        vh = {kk: v[p][slots[s]][None] for kk, v in pv.items()}
        ref = score.direct(k_method, qf[h], kh, kp, k_bits)
        compare_scores(got_s[h][:, :L], ref, score_tolerance(k_method, qf[h], kh, kp, k_bits), name="head %d" % h)
        assert np.all(got_s[h][:, L:] == sentinel)  # past the sequence's end: untouched
        ref_o = attention.decode(k_method, qf[h], kh, kp, k_bits, vh, vp, 3, 1.0 / np.sqrt(D))
        vmax = np.abs(attention.values_hat(vh, vp, 3, D)).max()
        err = np.abs(got_o[h] - ref_o)
        tol = attention_tolerance(ref_o, vmax, 1e-2)
        assert np.all(err <= tol), "attention head %d: max excess %g" % (h, float((err - tol).max()))
    pc.close()


def test_paged_identity_table_equals_contiguous():
    """Pages handed out in order to one sequence per head group: the paged calls give the unpaged calls'
    scores bit for bit (the same tiles, decoded the same way)."""
    page_tokens, L, kv_heads = 128, 1000, 2
    n_pages = -(-L // page_tokens)
    kp, vp, pi, T = _params("tq_prod", 3)
    pools = _pools("tq_prod", 3, 3, kv_heads, n_pages * page_tokens, seed=3)
    q = torch.randn((kv_heads, 8, D), generator=torch.Generator().manual_seed(1)).to(torch.float16).cuda()
    bt = torch.arange(n_pages, dtype=torch.int32).view(1, n_pages).cuda()
    sl = torch.tensor([L], dtype=torch.int32, device="cuda")
    c = _dev(kp["centroids"].astype(np.float32))
    kw = dict(pi=pi.cuda(), T=T.cuda(), signs=_dev(pools["k_signs"]), gammas=_dev(pools["k_gammas"]))
    a = kvrq.kv_score_packed_paged(kvrq.TQ_PROD, q, _dev(pools["k_words"]), _dev(pools["k_norms"]), 3, bt, sl,
                                   page_tokens, 1, kv_heads, L, c, **kw)
    b = kvrq.kv_score_packed(kvrq.TQ_PROD, q, _dev(pools["k_words"]), _dev(pools["k_norms"]), 3, L, c, **kw)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


@pytest.mark.parametrize("method,bits,dt", [("rq", 3, torch.float16), ("tq_mse", 3, torch.bfloat16),
                                            ("tq_prod", 3, torch.float16)])
def test_append_rows_into_pages(method, bits, dt):
    """One new vector per (layer, sequence, KV head) quantized into the slot the page manager gives the
    sequence's next token; the pool rows written equal the oracle's quantization of the new vectors, and no
    other row changes."""
    layers, kv_heads, lens, P = 2, 2, [5, 33, 16], 16
    pc, bt, slots, n_slots = _build_pages(P, lens, chunk=7, seed=1)
    seqs = list(range(len(lens)))
    new = [pc.append(s, 1) for s in seqs]  # first new logical token of each sequence
    new_slot = [int(pc.slots(s, t, 1)[0]) for s, t in zip(seqs, new)]
    pool_heads = layers * kv_heads
    rows = []  # (layer, seq, kv head) order, as the heads of a call
    for layer in range(layers):
        for s in seqs:
            for k in range(kv_heads):
                rows.append((layer * kv_heads + k) * n_slots + new_slot[s])
    n = len(rows)
    dst = torch.tensor(rows, dtype=torch.int64, device="cuda")
    x = (torch.randn((n, D), generator=torch.Generator().manual_seed(5)) *
         torch.exp(0.5 * torch.randn((n, 1), generator=torch.Generator().manual_seed(6)))).to(dt)
    cb_bits = bits - 1 if method == "tq_prod" else bits
    c64 = codebook.lloyd_max(D, cb_bits)[0].astype(np.float32).astype(np.float64)
    c = torch.from_numpy(c64.astype(np.float32)).cuda()
    ncode = 129 if method == "rq" else D
    W = kvrq.packed_words(ncode, cb_bits)
    canary = 0x5A5A5A5A
    codes = torch.full((pool_heads * n_slots, W), canary, dtype=torch.int32, device="cuda")
    norms = torch.full((pool_heads * n_slots,), -1.0, dtype=torch.float32, device="cuda")
    kw = {}
    pi = torch.from_numpy(params.rotation(D, 2)).to(dt)
    T = torch.from_numpy(params.qjl_matrix(D, D, 3)).to(torch.float16)
    if method == "rq":
        rot = params.rotors(D, 1).astype(np.float32)
        kw["rotors"] = torch.from_numpy(rot).cuda()
    else:
        kw["pi"] = pi.cuda()
    if method == "tq_prod":
        signs = torch.full((pool_heads * n_slots, D // 32), canary, dtype=torch.int32, device="cuda")
        gammas = torch.full((pool_heads * n_slots,), -1.0, dtype=torch.float32, device="cuda")
        kw.update(T=T.cuda(), signs=signs, gammas=gammas)
    m = {"rq": kvrq.RQ_MSE, "tq_mse": kvrq.TQ_MSE, "tq_prod": kvrq.TQ_PROD}[method]
    kvrq.kv_cache_append_rows(m, x.cuda(), dst, bits, c, codes, norms, **kw)
    torch.cuda.synchronize()
    kvrq.device_status()
    x64 = to_f64(x)
    got_c = words_u32(codes)[rows]
    if method == "rq":
        ref = rq.quantize(x64, rot.astype(np.float64), c64, bits)
    elif method == "tq_mse":
        ref = tq.mse_quantize(x64, pi.double().numpy(), c64, bits)
    else:
        ref = tq.prod_quantize(x64, pi.double().numpy(), T.double().numpy(), c64, bits)
    nb, bad = compare_codes(got_c, ref, ncode, cb_bits, c64)
    assert np.allclose(to_f64(norms)[rows], ref["norms"], rtol=1e-5)
    if method == "tq_prod":
        compare_sketch_signs(words_u32(signs)[rows], ref, x64, pi.double().numpy(), T.double().numpy(), c64,
                             skip_rows=bad)
        assert np.allclose(to_f64(gammas)[rows][~bad], ref["gammas"][~bad], rtol=1e-4, atol=1e-7)
    others = np.setdiff1d(np.arange(pool_heads * n_slots), rows)
    assert np.all(words_u32(codes)[others] == canary) and np.all(to_f64(norms)[others] == -1.0)
    pc.close()
