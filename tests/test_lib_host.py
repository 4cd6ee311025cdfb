"""Host-side checks of libkvrq.so (no GPU): symbols, parameter setup parity
against the oracle, and argument validation that must fail before any launch."""

import ctypes
import os
import re

import numpy as np
import pytest

import kv_cache_vector_rq_b200 as kvrq
from kv_cache_vector_rq_b200 import _lib
from oracle import codebook, params, rng

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
INCLUDE = os.path.join(ROOT, "include")


def _declared_functions():
    names = []
    for fname in sorted(os.listdir(INCLUDE)):
        if not fname.endswith(".h"):
            continue
        src = open(os.path.join(INCLUDE, fname)).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        src = re.sub(r"//[^\n]*", "", src)
        for m in re.finditer(r"^[A-Za-z_][\w \*]*?\b([A-Za-z_]\w*)\s*\(", src, flags=re.M):
            if m.group(1) not in ("if", "defined"):
                names.append(m.group(1))
    return names


def test_library_loads_and_exports_every_declared_symbol():
    lib = kvrq.lib()
    declared = _declared_functions()
    assert len(declared) >= 12
    for name in declared:
        assert hasattr(lib, name), "libkvrq.so does not export %s" % name
        assert name in _lib.SIGNATURES, "no ctypes signature for %s" % name
    assert set(_lib.SIGNATURES) == set(declared)
    assert "sm_100a" in kvrq.version()


def test_packed_words_and_groups():
    assert kvrq.packed_words(129, 3) == 13
    assert kvrq.packed_words(128, 3) == 12
    assert kvrq.packed_words(128, 2) == 8
    assert kvrq.packed_words(0, 3) == 0
    assert kvrq.rq_groups(128) == 43 and kvrq.rq_groups(3) == 1 and kvrq.rq_groups(4096) == 1366


# ------------------------------------------------------------------ setup parity

def test_normals_match_oracle_stream():
    for seed in (0, 1, 12345, 2 ** 63 + 7):
        a = kvrq.normals(seed, 0, 1001)
        b = rng.normals(seed, 1001)
        assert np.abs(a - b).max() < 1e-13
    # counter-based: any window of the stream
    assert np.abs(kvrq.normals(5, 37, 10) - rng.normals(5, 47)[37:]).max() < 1e-13


@pytest.mark.parametrize("d", [2, 3, 16, 64, 128, 129, 256, 1536, 4096])
@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_codebook_matches_oracle(d, bits):
    # Both sides iterate to max |change| < 1e-14 from different starts and evaluate
    # the cell integrals by different routes (continued fraction vs scipy), so they
    # agree to the fixed point's conditioning: ~1e-12 absolute, ~1e-10 relative at d = 4096.
    c_lib, t_lib = kvrq.tq_codebook_init(d, bits, tol=1e-14)
    c_or, t_or, _ = codebook.lloyd_max(d, bits, tol=1e-14)
    assert np.all(np.abs(c_lib - c_or) <= 1e-12 + 2e-10 * np.abs(c_or))
    assert np.all(np.abs(t_lib - t_or) <= 1e-12 + 2e-10 * np.abs(t_or))
    assert np.array_equal(c_lib, -c_lib[::-1])


def test_codebook_reports_non_convergence():
    c = np.zeros(8)
    st = kvrq.lib().tq_codebook_init(128, 3, 1e-15, 3, kvrq._dptr(c), None, None)
    assert st == 4  # KVRQ_ENOCONV


@pytest.mark.parametrize("d", [1, 2, 3, 4, 128, 4096])
def test_rotors_match_oracle(d):
    assert np.abs(kvrq.rq_rotors_init(d, 11) - params.rotors(d, 11)).max() < 1e-14


@pytest.mark.parametrize("d", [1, 2, 3, 17, 128, 256])
def test_rotation_matches_oracle(d):
    p_lib = kvrq.tq_rotation_init(d, 2)
    p_or = params.rotation(d, 2)
    assert np.abs(p_lib - p_or).max() < 1e-12
    assert np.abs(p_lib @ p_lib.T - np.eye(d)).max() < 1e-13


@pytest.mark.slow
def test_rotation_matches_oracle_large():
    p_lib = kvrq.tq_rotation_init(1536, 2)
    p_or = params.rotation(1536, 2)
    assert np.abs(p_lib - p_or).max() < 1e-11


def test_qjl_matrix_matches_oracle():
    assert np.abs(kvrq.qjl_matrix_init(128, 96, 3) - params.qjl_matrix(128, 96, 3)).max() < 1e-13


def test_setup_rejects_bad_arguments():
    lib = kvrq.lib()
    buf = np.zeros(64)
    assert lib.tq_codebook_init(1, 3, 1e-12, 100, kvrq._dptr(buf), None, None) == 1
    assert lib.tq_codebook_init(128, 0, 1e-12, 100, kvrq._dptr(buf), None, None) == 1
    assert lib.tq_codebook_init(128, 3, 0.0, 100, kvrq._dptr(buf), None, None) == 1
    assert lib.rq_rotors_init(0, 1, kvrq._dptr(buf)) == 1
    assert lib.tq_rotation_init(0, 1, kvrq._dptr(buf)) == 1
    assert lib.qjl_matrix_init(0, 4, 1, kvrq._dptr(buf)) == 1
    assert "d must be" in lib.kvrq_last_error_string().decode() or lib.kvrq_last_error_string()


# ------------------------------------------------------------------ hot-path validation (no launch)

P = 0x10000  # a fake, 16-byte aligned device address: validation fails before it is used


def test_rq_validation_fails_before_any_launch():
    lib = kvrq.lib()
    EINVAL, EUNSUP = 1, 2
    ok_args = dict(x=P, dt=1, n=10, d=128, ldx=128, rot=P, cb=P, bits=3, codes=P, ldc=13, norms=P)

    def q(**kw):
        a = dict(ok_args, **kw)
        return lib.rq_quantize(None, a["x"], a["dt"], a["n"], a["d"], a["ldx"], a["rot"], a["cb"], a["bits"],
                               a["codes"], a["ldc"], a["norms"])

    assert q(n=-1) == EINVAL
    assert q(d=1) == EINVAL
    assert q(bits=0) == EUNSUP and q(bits=5) == EUNSUP
    assert q(dt=7) == EINVAL
    assert q(x=None) == EINVAL
    assert q(rot=None) == EINVAL
    assert q(rot=P + 4) == EINVAL  # rotors must be 16-byte aligned
    assert q(ldx=100) == EINVAL
    assert q(ldc=12) == EINVAL  # 129 codes at 3 bits need 13 words
    assert q(codes=None) == EINVAL
    assert q(x=P + 1) == EINVAL  # not even element aligned
    assert q(n=0) == 0  # empty input is a no-op, no device touched
    msg = lib.kvrq_last_error_string().decode()
    assert isinstance(msg, str)
    # dequantize and fused calls share the same checks
    assert lib.rq_dequantize(None, P, 12, P, 10, 128, P, P, 3, P, 1, 128) == EINVAL
    assert lib.rq_dequantize(None, P, 13, P, 10, 128, P, P, 3, P, 9, 128) == EINVAL
    assert lib.rq_dequantize(None, P, 13, P, 0, 128, P, P, 3, P, 1, 128) == 0
    assert lib.rq_quantize_dequantize(None, P, 1, 10, 128, 128, P, P, 3, P, 13, P, None, 128) == EINVAL
    assert lib.rq_quantize_dequantize(None, P, 1, 10, 128, 128, P, P, 3, P, 13, P, P, 64) == EINVAL
    # the four-grade layout: 172 codes at d = 128 (17 words at 3 bits), d = 128 only
    assert lib.rq4_quantize(None, P, 1, 10, 128, 128, P, P, 3, P, 16, P) == EINVAL
    assert lib.rq4_quantize(None, P, 1, 10, 64, 64, P, P, 3, P, 17, P) == EUNSUP
    assert lib.rq4_quantize(None, P, 1, 0, 64, 64, P, P, 3, P, 17, P) == EUNSUP
    assert lib.rq4_quantize(None, P, 1, 0, 128, 128, P, P, 3, P, 17, P) == 0
    assert lib.rq4_dequantize(None, P, 16, P, 10, 128, P, P, 3, P, 1, 128) == EINVAL
    assert lib.rq4_dequantize(None, P, 11, P, 10, 128, P, P, 2, P, 1, 127) == EINVAL
    assert lib.rq4_quantize_dequantize(None, P, 1, 10, 128, 128, P, P, 4, P, 21, P, P, 128) == EINVAL
    assert kvrq.packed_words(172, 3) == 17 and kvrq.packed_words(172, 2) == 11 and kvrq.packed_words(172, 4) == 22


def test_tq_validation_fails_before_any_launch():
    lib = kvrq.lib()
    EINVAL, EUNSUP = 1, 2
    per_row = 4 * 256 + 4 * 2
    assert lib.kvrq_tq_workspace_bytes(1, 256) == per_row
    assert lib.kvrq_tq_workspace_bytes(0, 256) == 0

    def prod(d=256, m=256, ws=P, wsb=per_row * 128, n=10, dt=1, bits=3, ldc=None):
        W = -(-d * (bits - 1) // 32)
        return lib.tq_quantize_prod(None, P, dt, n, d, d, P, P, m, P, bits, P, W if ldc is None else ldc, P, m // 32,
                                    P, P, ws, wsb)

    assert prod(ws=None) == EINVAL  # the tiled prod path needs a workspace
    assert prod(wsb=per_row * 127) == EINVAL  # fewer than 128 rows fit
    assert prod(ws=P + 8) == EINVAL  # not 16-byte aligned
    assert prod(d=192, m=192) == EUNSUP  # not a multiple of 128
    assert prod(m=128) == EUNSUP  # m = d
    assert prod(bits=6) == EUNSUP
    assert prod(ldc=1) == EINVAL
    assert prod(n=0) == 0
    # d = 128 with 16-bit vectors takes no workspace; fp32 vectors do
    assert prod(d=128, m=128, ws=None, wsb=0, n=0) == 0
    assert prod(d=128, m=128, dt=0, ws=None, wsb=0) == EINVAL
    # dequantize: same workspace rule for prod, none for mse
    assert lib.tq_dequantize(None, P, 16, P, 8, P, P, 10, 256, 256, 3, P, P, P, P, 1, 256, None, 0) == EINVAL

    def sk(n=10, d=256, ldr=256, m=256, lds=8, dt=1):
        return lib.qjl_sketch(None, P, dt, n, d, ldr, P, m, P, lds, P, 1)

    assert sk(m=96) == EUNSUP
    assert sk(d=100, ldr=100) == EUNSUP
    assert sk(lds=7) == EINVAL
    assert sk(ldr=200) == EINVAL
    assert sk(n=-1) == EINVAL
    assert sk(n=0) == 0


def test_attention_chunk_count_stays_within_the_merge_limit():
    """The merge kernel holds at most 1,024 partials per query row: whatever the head count and length, the
    workspace is rows x 4 x (260 + chunks x 134) bytes with 1 <= chunks <= 1,024, and chunks covers the
    tokens (at least one 128-token tile per chunk of the tensor-core path, at most 1,024 of them)."""
    lib = kvrq.lib()
    for heads in (1, 3, 72, 148, 1152, 65535):
        for tokens in (1, 127, 128, 129, 4097, 131073, 1000000, 20000000):
            b = lib.kvrq_attention_workspace_bytes(heads, 8, tokens)
            per_row = b // (heads * 8 * 4)
            assert b == heads * 8 * 4 * per_row and (per_row - 260) % 134 == 0
            chunks = (per_row - 260) // 134
            assert 1 <= chunks <= 1024, (heads, tokens, chunks)


def test_attention_workspace_and_validation_fail_before_any_launch():
    lib = kvrq.lib()
    EINVAL, EUNSUP = 1, 2
    # rows x (132 rotated-query floats + 128 sketch floats + chunks x (132 sums + max + sum)) x 4 bytes, with
    # chunks the larger of the CUDA-core kernel's (token chunks of a multiple of 256 tokens) and the tensor-core
    # kernel's (one partial per work item: items of k 128-token tiles, k making ceil(items / 444) * (k + 1)
    # smallest for 444 warpgroup workers, at most 1,024 items per head)
    assert lib.kvrq_attention_workspace_bytes(1, 8, 1000) == 8 * 4 * (260 + 8 * 134)  # 8 items of 128 tokens
    # 33 CUDA-core chunks of 4,096 tokens (the tensor-core path: 6 items of 171 tiles)
    assert lib.kvrq_attention_workspace_bytes(72, 8, 131073) == 576 * 4 * (260 + 33 * 134)
    # 977 CUDA-core chunks of 1,024 tokens (the tensor-core path: 435 items of 18 tiles)
    assert lib.kvrq_attention_workspace_bytes(1, 1, 1000000) == 4 * (260 + 977 * 134)
    assert lib.kvrq_attention_workspace_bytes(0, 8, 100) == 0
    wsb = lib.kvrq_attention_workspace_bytes(2, 8, 100)

    def att(method=0, n_heads=2, group=8, d=128, scale=0.088, k_bits=3, m=128, ldk=13, ldv=13, n_tokens=100,
            ws=P, wsb=wsb, kr=P, vr=P, pi=None, T=None, ks=None, kg=None, qdt=1, odt=0, tok=100):
        return lib.kv_attention_packed(None, method, P, qdt, 128, n_heads, group, d, scale, k_bits, m, P, ldk,
                                       ldk * 100, ks, 4, 400, P, kg, kr, pi, 1, T, P, P, ldv, ldv * 100, P, 3, vr, P,
                                       tok, n_tokens, P, odt, 128, ws, wsb)

    assert att(method=7) == EINVAL
    assert att(d=64) == EUNSUP
    assert att(group=17) == EUNSUP and att(group=0) == EINVAL
    assert att(k_bits=5) == EUNSUP
    assert att(method=2, k_bits=1, pi=P, T=P, ks=P, kg=P) == EUNSUP  # prod stores k_bits - 1 >= 1 bits
    assert att(method=2, m=64, pi=P, T=P, ks=P, kg=P) == EUNSUP
    assert att(qdt=9) == EINVAL and att(odt=9) == EINVAL
    assert att(scale=float("nan")) == EINVAL
    assert att(n_heads=0) == 0  # no-op
    assert att(n_tokens=0) == EINVAL  # softmax over no tokens
    assert att(ldk=12) == EINVAL  # 129 codes at 3 bits need 13 words
    assert att(ldv=12) == EINVAL
    assert att(tok=99) == EINVAL
    assert att(kr=None) == EINVAL and att(kr=P + 4) == EINVAL
    assert att(vr=P + 8) == EINVAL
    assert att(method=1, ldk=12) == EINVAL  # TurboQuant keys need pi
    assert att(method=2, ldk=8, pi=P, T=P) == EINVAL  # prod needs signs and gammas
    assert att(ws=None) == EINVAL and att(wsb=wsb - 4) == EINVAL and att(ws=P + 4) == EINVAL
    assert att(n_heads=70000, wsb=1 << 40) == EUNSUP


def test_score_and_append_validation_fail_before_any_launch():
    lib = kvrq.lib()
    EINVAL, EUNSUP = 1, 2

    def sc(method=0, n_heads=4, group=8, d=128, bits=3, m=128, ldc=13, chs=13 * 100, lds=4, shs=400, tok=100,
           n_tokens=100, rot=P, pi=None, pdt=1, T=None, signs=None, gam=None, qdt=1, ldq=128, lsc=100, codes=P):
        return lib.kv_score_packed(None, method, P, qdt, ldq, n_heads, group, d, bits, m, codes, ldc, chs, signs,
                                   lds, shs, P, gam, tok, n_tokens, rot, pi, pdt, T, P, P, lsc)

    assert sc(method=5) == EINVAL
    assert sc(group=0) == EINVAL and sc(n_tokens=-1) == EINVAL
    assert sc(d=256) == EUNSUP
    assert sc(bits=5) == EUNSUP and sc(method=2, bits=1, pi=P, T=P, signs=P, gam=P, ldc=4) == EUNSUP
    assert sc(group=65) == EUNSUP and sc(method=2, group=33, pi=P, T=P, signs=P, gam=P, ldc=8) == EUNSUP
    assert sc(method=2, m=64, pi=P, T=P, signs=P, gam=P, ldc=8) == EUNSUP  # the sketch needs m = d
    assert sc(qdt=4) == EINVAL and sc(ldq=100) == EINVAL
    assert sc(n_heads=0) == 0 and sc(n_tokens=0) == 0  # no-ops
    assert sc(codes=None) == EINVAL
    assert sc(ldc=12) == EINVAL and sc(chs=1299) == EINVAL and sc(tok=99) == EINVAL and sc(lsc=99) == EINVAL
    assert sc(rot=None) == EINVAL and sc(rot=P + 4) == EINVAL
    assert sc(method=1, ldc=12) == EINVAL  # TurboQuant keys need pi
    assert sc(method=1, ldc=12, pi=P, pdt=0) == EINVAL  # pi must be fp16 or bf16
    assert sc(method=2, ldc=8, pi=P, T=P) == EINVAL  # prod needs signs and gammas
    assert sc(method=2, ldc=8, pi=P, T=P, signs=P, gam=P, lds=3) == EINVAL
    assert sc(n_heads=70000, chs=1300) == EUNSUP

    def ap(method=0, n=8, d=128, ldx=128, bits=3, ldc=13, lnr=1, codes=P, rot=P):
        return lib.kv_cache_append(None, method, P, 1, n, d, ldx, bits, rot, None, None, 128, P, codes, ldc, None, 0,
                                   P, None, lnr)

    assert ap(method=9) == EINVAL
    assert ap(bits=5) == EUNSUP
    assert ap(ldc=12) == EINVAL  # a code row of 129 codes at 3 bits needs 13 words
    assert ap(lnr=0) == EINVAL
    assert ap(rot=None) == EINVAL
    assert ap(n=0) == 0

    # the no-allocation prod quantize shares the prod checks and rejects a block that does not fit its array
    def na(d=256, m=256, n=10, bits=3):
        W = -(-d * (bits - 1) // 32)
        return lib.tq_quantize_prod_noalloc(None, P, 1, n, d, d, P, P, m, P, bits, P, W, P, m // 32, P, P)

    assert na(d=16384, m=16384) == EUNSUP
    assert na(m=128) == EUNSUP
    assert na(bits=6) == EUNSUP


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    # no fallback path: without libkvrq.so the binding refuses to load, and every call goes through it
    monkeypatch.setattr(_lib, "_lib", None)
    monkeypatch.setattr(_lib, "LIB_PATH", str(tmp_path / "libkvrq.so"))
    with pytest.raises(ImportError, match="not built"):
        kvrq.lib()
    with pytest.raises(ImportError):
        kvrq.packed_words(129, 3)


@pytest.mark.parametrize("level,bits", [(1, 4), (2, 2), (3, 2), (4, 2), (2, 3), (3, 4)])
def test_polar_angle_codebook_matches_oracle(level, bits):
    from oracle import polar

    c, t = kvrq.pq_angle_codebook_init(level, bits)
    co, _ = polar.lloyd_max_angles(level, bits)
    np.testing.assert_allclose(c, co, rtol=0, atol=1e-12)
    np.testing.assert_allclose(t, 0.5 * (c[:-1] + c[1:]), rtol=0, atol=0)
    if level >= 2:
        np.testing.assert_allclose(c + c[::-1], np.pi / 2, rtol=0, atol=1e-15)  # symmetric about pi/4


def test_polar_angle_codebook_errors():
    lib = kvrq.lib()
    c = np.zeros(16)
    it = ctypes.c_int(0)
    dp = lambda a: a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))
    assert lib.pq_angle_codebook_init(0, 2, 1e-13, 100, dp(c), None, None) == 1
    assert lib.pq_angle_codebook_init(2, 9, 1e-13, 100, dp(c), None, None) == 1
    assert lib.pq_angle_codebook_init(2, 2, 0.0, 100, dp(c), None, None) == 1
    assert lib.pq_angle_codebook_init(2, 2, 1e-13, 100, None, None, None) == 1
    assert lib.pq_angle_codebook_init(2, 2, 1e-13, 1, dp(c), None, ctypes.byref(it)) == 4  # KVRQ_ENOCONV
    assert it.value == 1
