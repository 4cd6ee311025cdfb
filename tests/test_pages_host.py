"""Paged KV-cache bookkeeping (kvrq_pages_*), on the CPU: random add / append / free sequences
checked against the definition (token t of a sequence is slot P * table[t // P] + t % P), page
conservation, disjoint tables, all-or-nothing appends, errors, and concurrent appends."""

import threading

import numpy as np
import pytest

import kv_cache_vector_rq_b200 as kvrq
from kv_cache_vector_rq_b200 import KvrqError


def _check(pc, n_pages, P, model):
    used = []
    all_slots = []
    for sid, length in model.items():
        table, n_tok = pc.block_table(sid)
        assert n_tok == length
        assert len(table) == -(-length // P)
        used.extend(table.tolist())
        slots = pc.slots(sid, 0, length)
        t = np.arange(length)
        np.testing.assert_array_equal(slots, table[t // P].astype(np.int64) * P + t % P)
        all_slots.extend(slots.tolist())
    assert len(set(used)) == len(used)  # no page in two tables
    assert all(0 <= p < n_pages for p in used)
    assert len(set(all_slots)) == len(all_slots)
    free, n_seqs = pc.stats()
    assert free + len(used) == n_pages and n_seqs == len(model)


@pytest.mark.parametrize("n_pages,P,seed", [(64, 16, 0), (500, 7, 1), (8, 1, 2)])
def test_random_operations(n_pages, P, seed):
    g = np.random.default_rng(seed)
    pc = kvrq.PagedCache(n_pages, P)
    model = {}
    for step in range(400):
        op = g.random()
        if op < 0.2 or not model:
            model[pc.add_seq()] = 0
        elif op < 0.85:
            sid = list(model)[g.integers(len(model))]
            n = int(g.integers(0, 3 * P + 2))
            free_before = pc.stats()[0]
            need = -(-(model[sid] + n) // P) - (-(-model[sid] // P))
            if need > free_before:
                with pytest.raises(KvrqError):
                    pc.append(sid, n)
                assert pc.stats()[0] == free_before  # nothing reserved
            else:
                assert pc.append(sid, n) == model[sid]
                model[sid] += n
        else:
            sid = list(model)[g.integers(len(model))]
            pc.free_seq(sid)
            del model[sid]
        if step % 25 == 0:
            _check(pc, n_pages, P, model)
    _check(pc, n_pages, P, model)
    pc.close()


def test_first_pages_and_reuse():
    pc = kvrq.PagedCache(4, 8)
    a = pc.add_seq()
    assert pc.append(a, 10) == 0
    table, n = pc.block_table(a)
    assert table.tolist() == [0, 1] and n == 10
    np.testing.assert_array_equal(pc.slots(a, 8, 2), [8, 9])
    b = pc.add_seq()
    assert b != a
    pc.append(b, 1)
    assert pc.block_table(b)[0].tolist() == [2]
    pc.free_seq(a)
    c = pc.add_seq()
    pc.append(c, 16)
    assert sorted(pc.block_table(c)[0].tolist()) == [0, 1]  # a's pages are handed out again


def test_errors():
    with pytest.raises(KvrqError):
        kvrq.PagedCache(0, 4)
    with pytest.raises(KvrqError):
        kvrq.PagedCache(4, 0)
    pc = kvrq.PagedCache(2, 4)
    s = pc.add_seq()
    with pytest.raises(KvrqError):
        pc.append(s, 9)  # three pages needed, two exist
    with pytest.raises(KvrqError):
        pc.append(s + 100, 1)
    pc.append(s, 3)
    with pytest.raises(KvrqError):
        pc.slots(s, 2, 2)  # token 3 is past the end
    with pytest.raises(KvrqError):
        pc.free_seq(s + 1)
    pc.free_seq(s)
    with pytest.raises(KvrqError):
        pc.free_seq(s)  # ids are not reused
    kvrq.lib().kvrq_pages_destroy(None)  # no-op


def test_overflow_guards():
    """Counts near INT64_MAX are rejected before any arithmetic can wrap: slots() with a huge count must not
    read past the block table, append() with a huge n_tokens must not reserve anything."""
    import ctypes
    big = (1 << 63) - 1
    pc = kvrq.PagedCache(4, 8)
    s = pc.add_seq()
    pc.append(s, 10)
    buf = np.full(4, -7, dtype=np.int64)
    ptr = buf.ctypes.data_as(ctypes.c_void_p)
    for first, count in ((1, big), (10, big - 9), (big, 1), (11, 0), (0, 11)):
        assert kvrq.lib().kvrq_pages_slots(pc._h, s, first, count, ptr) == 1  # KVRQ_EINVAL
    assert np.all(buf == -7)  # nothing written
    assert kvrq.lib().kvrq_pages_slots(pc._h, s, 10, 0, ptr) == 0  # an empty range at the end is fine
    for n in (big, big - 10, big - 17):
        with pytest.raises(KvrqError):
            pc.append(s, n)
    table, n_tok = pc.block_table(s)
    assert n_tok == 10 and len(table) == 2 and pc.stats()[0] == 2  # nothing reserved
    pc.close()


def test_concurrent_appends():
    pc = kvrq.PagedCache(4096, 8)
    seqs = [pc.add_seq() for _ in range(16)]

    def work(sid):
        for _ in range(200):
            pc.append(sid, 1)

    threads = [threading.Thread(target=work, args=(s,)) for s in seqs]
    for t in threads:
        t.start()
    for t in threads:
        t.join()
    _check(pc, 4096, 8, {s: 200 for s in seqs})
