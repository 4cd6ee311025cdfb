"""Host failure paths, on the CPU: allocation failures injected through the library's test hook, parameter
files with a corrupted payload or checksum, and the paged calls' argument checks. Each failing call must
return its status, explain it, and change nothing."""

import ctypes

import numpy as np
import pytest

import kv_cache_vector_rq_b200 as kvrq
from kv_cache_vector_rq_b200 import KvrqError, _lib

ENOMEM, ECHECKSUM, EINVAL, EUNSUP = 6, 7, 1, 2
P = 1 << 20  # a plausible, 16-byte aligned device address: argument checks fail before any launch


@pytest.fixture(autouse=True)
def _disarm():
    yield
    kvrq.lib().kvrq_test_fail_allocations(0)


def _last_error():
    return kvrq.lib().kvrq_last_error_string().decode()


def test_allocation_failure_in_parameter_setup():
    lib = kvrq.lib()
    c = np.zeros(8)
    lib.kvrq_test_fail_allocations(1)
    st = lib.tq_codebook_init(128, 3, 1e-13, 100000, c.ctypes.data_as(ctypes.POINTER(ctypes.c_double)), None, None)
    assert st == ENOMEM and "memory" in _last_error()
    assert np.all(c == 0)  # nothing written
    # the hook is spent: the same call succeeds and equals the plain result
    c2, _ = kvrq.tq_codebook_init(128, 3)
    assert lib.tq_codebook_init(128, 3, 1e-13, 100000, c.ctypes.data_as(ctypes.POINTER(ctypes.c_double)), None, None) == 0
    assert np.array_equal(c, c2)
    pi = np.zeros((64, 64))
    lib.kvrq_test_fail_allocations(1)
    assert lib.tq_rotation_init(64, 2, pi.ctypes.data_as(ctypes.POINTER(ctypes.c_double))) == ENOMEM and np.all(pi == 0)
    lib.kvrq_test_fail_allocations(1)
    cb = np.zeros(4)
    assert lib.pq_angle_codebook_init(2, 2, 1e-13, 1000, cb.ctypes.data_as(ctypes.POINTER(ctypes.c_double)), None, None) == ENOMEM


def test_allocation_failure_in_page_manager_changes_nothing():
    lib = kvrq.lib()
    h = ctypes.c_void_p()
    lib.kvrq_test_fail_allocations(1)
    assert lib.kvrq_pages_create(8, 4, ctypes.byref(h)) == ENOMEM and not h.value
    pc = kvrq.PagedCache(8, 4)
    s = pc.add_seq()
    pc.append(s, 5)  # two pages
    free0 = pc.stats()[0]
    table0, n0 = pc.block_table(s)
    lib.kvrq_test_fail_allocations(1)
    with pytest.raises(KvrqError):
        pc.append(s, 9)  # would need three more pages: the allocation fails first
    assert pc.stats()[0] == free0 and pc.block_table(s)[1] == n0
    assert np.array_equal(pc.block_table(s)[0], table0)
    lib.kvrq_test_fail_allocations(1)
    sid = ctypes.c_int64(-1)
    assert lib.kvrq_pages_add_seq(pc._h, ctypes.byref(sid)) == ENOMEM and sid.value == -1
    assert pc.stats()[1] == 1
    # after the failures the manager works on: the new sequence gets the next id, pages are consistent
    s2 = pc.add_seq()
    assert s2 == s + 1
    pc.append(s2, 8)
    assert pc.stats()[0] == free0 - 2
    pc.close()


def test_parameter_file_roundtrip_and_checksum(tmp_path):
    d, bits, m, seed = 96, 3, 64, 11
    path = tmp_path / "p.kvrq"
    kvrq.params_export(str(path), d, bits, m, seed)
    got = kvrq.params_import(str(path), d, bits, m)
    assert got["seed"] == seed
    assert np.array_equal(got["rotors"], kvrq.rq_rotors_init(d, seed + 1))
    assert np.array_equal(got["pi"], kvrq.tq_rotation_init(d, seed + 2))
    assert np.array_equal(got["T"], kvrq.qjl_matrix_init(m, d, seed + 3))
    assert np.array_equal(got["centroids"], kvrq.tq_codebook_init(d, bits)[0])
    raw = bytearray(path.read_bytes())
    header_end = raw.index(b"\n", raw.index(b"\n") + 1) + 1
    # one flipped payload bit: the checksum rejects the file, and no output is written
    bad = bytearray(raw)
    bad[header_end + 1000] ^= 0x10
    (tmp_path / "bad.kvrq").write_bytes(bytes(bad))
    rot = np.full((-(-d // 3), 4), 7.0)
    st = kvrq.lib().kvrq_params_import(str(tmp_path / "bad.kvrq").encode(), d, bits, m, None,
                                       rot.ctypes.data_as(ctypes.c_void_p), None, None, None)
    assert st == ECHECKSUM and "checksum" in _last_error() and np.all(rot == 7.0)
    # a tampered checksum in the header
    hdr = bytearray(raw)
    i = raw.index(b'"fnv1a64": "') + len(b'"fnv1a64": "')
    hdr[i] = ord("0") if hdr[i] != ord("0") else ord("1")
    (tmp_path / "hdr.kvrq").write_bytes(bytes(hdr))
    with pytest.raises(KvrqError, match="checksum"):
        kvrq.params_import(str(tmp_path / "hdr.kvrq"), d, bits, m)
    # truncated, another configuration, not a parameter file, a missing file
    (tmp_path / "short.kvrq").write_bytes(bytes(raw[:-8]))
    assert kvrq.lib().kvrq_params_import(str(tmp_path / "short.kvrq").encode(), d, bits, m, None, None, None, None,
                                         None) == EINVAL
    assert kvrq.lib().kvrq_params_import(str(path).encode(), d, 2, m, None, None, None, None, None) == EINVAL
    (tmp_path / "junk.kvrq").write_bytes(b"hello\n")
    assert kvrq.lib().kvrq_params_import(str(tmp_path / "junk.kvrq").encode(), d, bits, m, None, None, None, None,
                                         None) == EINVAL
    assert kvrq.lib().kvrq_params_import(str(tmp_path / "none.kvrq").encode(), d, bits, m, None, None, None, None,
                                         None) == EINVAL
    # an allocation failure while exporting writes no file
    kvrq.lib().kvrq_test_fail_allocations(1)
    assert kvrq.lib().kvrq_params_export(str(tmp_path / "oom.kvrq").encode(), d, bits, m, seed) == ENOMEM
    assert not (tmp_path / "oom.kvrq").exists()


def test_paged_calls_validate_before_any_launch():
    lib = kvrq.lib()
    tables = np.zeros((3, 8), dtype=np.int32)
    lens = np.zeros(3, dtype=np.int32)
    pg = _lib.KvrqPaged(P, 8, P, 16, 3, 2)

    def score(paged=ctypes.byref(pg), n_heads=12, max_tokens=128):
        return lib.kv_score_packed_paged(None, 2, P, 1, 128, n_heads, 8, 128, 3, 128, P, 8, 1000, P, 4, 1000, P, P,
                                         1000, paged, max_tokens, None, P, 1, P, P, P, max_tokens)

    assert score(paged=None) == EINVAL
    assert score(n_heads=10) == EINVAL  # not a multiple of n_seqs x kv_heads = 6
    assert score(max_tokens=200) == EINVAL  # ld_table 8 pages of 16 slots hold 128 tokens
    for bad in (_lib.KvrqPaged(0, 8, P, 16, 3, 2), _lib.KvrqPaged(P, 8, 0, 16, 3, 2), _lib.KvrqPaged(P, 8, P, 0, 3, 2),
                _lib.KvrqPaged(P, 8, P + 2, 16, 3, 2)):
        assert score(paged=ctypes.byref(bad)) == EINVAL

    def att(k_method=2, k_bits=3, v_bits=3, group=8, paged=ctypes.byref(pg)):
        ldv = -(-129 * v_bits // 32)
        return lib.kv_attention_packed_paged(None, k_method, P, 1, 128, 12, group, 128, 0.088, k_bits, 128, P, 8, 1000,
                                             P, 4, 1000, P, P, None, P, 1, P, P, P, ldv, 1000, P, v_bits, P, P, 1000,
                                             paged, 128, P, 0, 128, P, 1 << 30)

    assert att(paged=None) == EINVAL
    assert att(v_bits=4) == EUNSUP  # the paged cache is read by the tensor-core kernel only
    assert att(group=16) == EUNSUP
    # the append with destination rows: d = 128 only, rows required
    assert lib.kv_cache_append_rows(None, 0, P, 1, 4, 128, 128, 3, P, None, None, 128, P, None, P, 13, None, 0, P,
                                    None, 1) == EINVAL
    assert lib.kv_cache_append_rows(None, 0, P, 1, 4, 96, 96, 3, P, None, None, 96, P, P, P, 11, None, 0, P, None,
                                    1) == EUNSUP
    assert lib.kv_cache_append_rows(None, 1, P, 0, 4, 128, 128, 3, None, P, None, 128, P, P, P, 12, None, 0, P, None,
                                    1) == EUNSUP  # fp32 TurboQuant rows run the tiled kernel: no destination rows


def test_host_roundtrip_validates_before_anything_is_queued():
    """rq_quantize_dequantize_host checks its pointers, strides and workspace before it touches a device
    (these run without one): NULL host arrays, ldx below d, a misaligned or too small workspace."""
    lib = kvrq.lib()
    d, bits = 128, 3
    ws_min = lib.kvrq_host_workspace_bytes(d, bits, kvrq.F16, 32)
    assert ws_min > 0 and ws_min % 256 == 0
    assert lib.kvrq_host_workspace_bytes(d, bits, kvrq.F16, 33) == lib.kvrq_host_workspace_bytes(d, bits, kvrq.F16, 64)
    assert lib.kvrq_host_workspace_bytes(d, bits, kvrq.F16, 31) == 0  # below one 32-row chunk
    assert lib.kvrq_host_workspace_bytes(d, 5, kvrq.F16, 64) == 0
    big = lib.kvrq_host_workspace_bytes(d, bits, kvrq.F16, 4096)
    assert big > 100 * ws_min  # three slots of 4096 rows against three of 32
    fake = ctypes.c_void_p(1 << 20)  # never dereferenced: every call below fails its checks first
    args = dict(stream=None, x=fake, dt=kvrq.F16, n=100, d=d, ldx=d, rot=fake, cb=fake, bits=bits, codes=fake, ldc=13,
                norms=fake, xhat=fake, ldo=d, ws=fake, wsb=ws_min)

    def call(**kw):
        a = dict(args, **kw)
        return lib.rq_quantize_dequantize_host(a["stream"], a["x"], a["dt"], a["n"], a["d"], a["ldx"], a["rot"], a["cb"],
                                               a["bits"], a["codes"], a["ldc"], a["norms"], a["xhat"], a["ldo"],
                                               a["ws"], a["wsb"])
    assert call(x=None) == EINVAL
    assert call(xhat=None) == EINVAL
    assert call(ldx=d - 1) == EINVAL
    assert call(ldc=12) == EINVAL  # 129 3-bit codes need 13 words
    assert call(ws=ctypes.c_void_p((1 << 20) + 16)) == EINVAL  # not 256-byte aligned
    assert call(wsb=ws_min - 256) == EINVAL
    assert call(bits=5) == EUNSUP
    assert call(n=0) == 0  # nothing to do
