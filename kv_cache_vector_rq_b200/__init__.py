"""kvrq: B200-native online vector quantization of KV-cache vectors.

RotorQuant (Cl(3,0) rotor sandwich on 3-dim groups) and TurboQuant (dense
random rotation, Lloyd-Max, optional 1-bit QJL residual sketch) as
hand-written sm_100a CUDA kernels behind a C ABI (include/kvrq.h, libkvrq.so).

This module is a thin binding: it checks tensor placement, dtype and layout
and passes raw pointers to the library. Every step of the quantization runs
in the library's kernels; PyTorch only supplies device memory and streams.
Parameters (codebook, rotors, Pi, QJL matrix) are produced by the library's
host setup functions in float64 and returned as numpy arrays.
"""

import ctypes
import os

import numpy as np

from . import _lib
from ._lib import KvrqError

F32, F16, BF16 = 0, 1, 2
RQ_MSE, TQ_MSE, TQ_PROD = 0, 1, 2


def lib():
    return _lib.load()


def version():
    return lib().kvrq_version().decode()


def _dptr(a):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


# ----------------------------------------------------------------------------- setup (host)

def packed_words(n_codes, bits):
    return int(lib().kvrq_packed_words(n_codes, bits))


def rq_groups(d):
    return int(lib().kvrq_rq_groups(d))


def tq_codebook_init(d, bits, tol=1e-13, max_iter=100000):
    """Lloyd-Max centroids and boundaries (float64 numpy) for dimension d."""
    K = 1 << bits
    c = np.zeros(K)
    t = np.zeros(K - 1)
    it = ctypes.c_int(0)
    _lib.check("tq_codebook_init", lib().tq_codebook_init(d, bits, tol, max_iter, _dptr(c), _dptr(t), ctypes.byref(it)))
    return c, t


def pq_angle_codebook_init(level, bits, tol=1e-13, max_iter=100000):
    """PolarQuant angle centroids and boundaries (float64 numpy) of one polar-transform level."""
    K = 1 << bits
    c = np.zeros(K)
    t = np.zeros(K - 1)
    it = ctypes.c_int(0)
    _lib.check("pq_angle_codebook_init",
               lib().pq_angle_codebook_init(level, bits, tol, max_iter, _dptr(c), _dptr(t), ctypes.byref(it)))
    return c, t


def params_export(path, d, bits, m, seed):
    """Write the parameters of (d, bits, m, seed) to a checksummed file (kvrq_params_export)."""
    _lib.check("kvrq_params_export", lib().kvrq_params_export(os.fsencode(path), d, bits, m, seed))


def params_import(path, d, bits, m):
    """Read and verify a parameter file: returns dict(seed, rotors [G, 4], pi [d, d], T [m, d], centroids)."""
    G = rq_groups(d)
    out = {"rotors": np.zeros((G, 4)), "pi": np.zeros((d, d)), "T": np.zeros((m, d)), "centroids": np.zeros(1 << bits)}
    seed = ctypes.c_uint64(0)
    _lib.check("kvrq_params_import", lib().kvrq_params_import(
        os.fsencode(path), d, bits, m, ctypes.byref(seed), _dptr(out["rotors"]), _dptr(out["pi"]), _dptr(out["T"]),
        _dptr(out["centroids"])))
    out["seed"] = seed.value
    return out


def rq_rotors_init(d, seed):
    G = rq_groups(d)
    r = np.zeros((G, 4))
    _lib.check("rq_rotors_init", lib().rq_rotors_init(d, seed, _dptr(r)))
    return r


def tq_rotation_init(d, seed):
    p = np.zeros((d, d))
    _lib.check("tq_rotation_init", lib().tq_rotation_init(d, seed, _dptr(p)))
    return p


def qjl_matrix_init(m, d, seed):
    t = np.zeros((m, d))
    _lib.check("qjl_matrix_init", lib().qjl_matrix_init(m, d, seed, _dptr(t)))
    return t


def normals(seed, first, count):
    out = np.zeros(count)
    _lib.check("kvrq_normals", lib().kvrq_normals(seed, first, count, _dptr(out)))
    return out


# ----------------------------------------------------------------------------- device calls

def _torch():
    import torch

    return torch


def _dtype_code(t):
    torch = _torch()
    m = {torch.float32: F32, torch.float16: F16, torch.bfloat16: BF16}
    if t.dtype not in m:
        raise TypeError("unsupported dtype %s" % t.dtype)
    return m[t.dtype]


def _rows(t, name):
    """(pointer, leading dimension) of a 2-D CUDA tensor with unit inner stride."""
    if not t.is_cuda:
        raise ValueError("%s must be a CUDA tensor" % name)
    if t.dim() != 2 or (t.shape[1] > 1 and t.stride(1) != 1):
        raise ValueError("%s must be 2-D with unit column stride" % name)
    return t.data_ptr(), (t.stride(0) if t.shape[0] > 1 else t.shape[1])


def _ptr(t, name, dtype=None):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("%s must be a CUDA tensor" % name)
    if dtype is not None and t.dtype != dtype:
        raise TypeError("%s must be %s" % (name, dtype))
    return t.data_ptr()


def _stream(stream):
    torch = _torch()
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def rq_quantize(x, rotors, centroids, bits, codes=None, norms=None, stream=None, _fn="rq_quantize", _cpg=3):
    """Quantize rows of x [n, d] (fp32/fp16/bf16 CUDA). Returns (codes [n, W] int32 view of uint32, norms [n])."""
    torch = _torch()
    n, d = x.shape
    W = packed_words(_cpg * rq_groups(d), bits)
    if codes is None:
        codes = torch.empty((n, W), dtype=torch.int32, device=x.device)
    if norms is None:
        norms = torch.empty((n,), dtype=torch.float32, device=x.device)
    xp, ldx = _rows(x, "x")
    cp, ldc = _rows(codes, "codes")
    _lib.check(_fn, getattr(lib(), _fn)(_stream(stream), xp, _dtype_code(x), n, d, ldx,
                                        _ptr(rotors, "rotors", torch.float32),
                                        _ptr(centroids, "centroids", torch.float32), bits, cp, ldc,
                                        _ptr(norms, "norms", torch.float32)))
    return codes, norms


def rq_dequantize(codes, norms, d, rotors, centroids, bits, out_dtype=None, xhat=None, stream=None,
                  _fn="rq_dequantize"):
    """Dequantize packed codes [n, W] + norms [n] into x_hat [n, d]."""
    torch = _torch()
    n = codes.shape[0]
    if xhat is None:
        xhat = torch.empty((n, d), dtype=out_dtype or torch.float16, device=codes.device)
    cp, ldc = _rows(codes, "codes")
    op, ldo = _rows(xhat, "xhat")
    _lib.check(_fn, getattr(lib(), _fn)(_stream(stream), cp, ldc, _ptr(norms, "norms", torch.float32), n, d,
                                        _ptr(rotors, "rotors", torch.float32),
                                        _ptr(centroids, "centroids", torch.float32), bits, op,
                                        _dtype_code(xhat), ldo))
    return xhat


def rq_quantize_dequantize(x, rotors, centroids, bits, codes=None, norms=None, xhat=None, with_codes=True,
                           stream=None, _fn="rq_quantize_dequantize", _cpg=3):
    """Fused roundtrip: returns (codes, norms, x_hat); codes/norms are None when with_codes is False."""
    torch = _torch()
    n, d = x.shape
    W = packed_words(_cpg * rq_groups(d), bits)
    if with_codes and codes is None:
        codes = torch.empty((n, W), dtype=torch.int32, device=x.device)
    if with_codes and norms is None:
        norms = torch.empty((n,), dtype=torch.float32, device=x.device)
    if xhat is None:
        xhat = torch.empty_like(x)
    xp, ldx = _rows(x, "x")
    cp, ldc = _rows(codes, "codes") if codes is not None else (None, W)
    op, ldo = _rows(xhat, "xhat")
    _lib.check(_fn, getattr(lib(), _fn)(
        _stream(stream), xp, _dtype_code(x), n, d, ldx, _ptr(rotors, "rotors", torch.float32),
        _ptr(centroids, "centroids", torch.float32), bits, cp, ldc, _ptr(norms, "norms", torch.float32), op, ldo))
    return codes, norms, xhat


def host_workspace_bytes(d, bits, dtype, chunk_rows=4096):
    """Device workspace bytes of rq_quantize_dequantize_host for chunks of chunk_rows rows."""
    torch = _torch()
    code = {torch.float32: F32, torch.float16: F16, torch.bfloat16: BF16}[dtype]
    return int(lib().kvrq_host_workspace_bytes(d, bits, code, chunk_rows))


def _host_rows(t, name):
    """(pointer, leading dimension) of a 2-D host tensor with unit inner stride."""
    if t.is_cuda:
        raise ValueError("%s must be a host tensor" % name)
    if t.dim() != 2 or (t.shape[1] > 1 and t.stride(1) != 1):
        raise ValueError("%s must be 2-D with unit column stride" % name)
    return t.data_ptr(), (t.stride(0) if t.shape[0] > 1 else t.shape[1])


def rq_quantize_dequantize_host(x, rotors, centroids, bits, workspace, codes=None, norms=None, xhat=None,
                                stream=None):
    """Fused roundtrip of host rows x [n, d] (ideally pinned) through the device, in chunks whose copy-in, kernel
    and copy-out overlap: returns host (codes [n, W], norms [n], x_hat [n, d]) (pinned when allocated here).
    workspace: a CUDA tensor of at least host_workspace_bytes(d, bits, x.dtype, 32) bytes. Asynchronous on
    `stream`, like the device calls: synchronize before reading the outputs."""
    torch = _torch()
    n, d = x.shape
    W = packed_words(3 * rq_groups(d), bits)
    if codes is None:
        codes = torch.empty((n, W), dtype=torch.int32).pin_memory()
    if norms is None:
        norms = torch.empty((n,), dtype=torch.float32).pin_memory()
    if xhat is None:
        xhat = torch.empty((n, d), dtype=x.dtype).pin_memory()
    if not workspace.is_cuda:
        raise ValueError("workspace must be a CUDA tensor")
    xp, ldx = _host_rows(x, "x")
    cp, ldc = _host_rows(codes, "codes")
    op, ldo = _host_rows(xhat, "xhat")
    if norms.is_cuda or not norms.is_contiguous() or norms.dtype != torch.float32:
        raise ValueError("norms must be a contiguous fp32 host tensor")
    _lib.check("rq_quantize_dequantize_host", lib().rq_quantize_dequantize_host(
        _stream(stream), xp, _dtype_code(x), n, d, ldx, _ptr(rotors, "rotors", torch.float32),
        _ptr(centroids, "centroids", torch.float32), bits, cp, ldc, norms.data_ptr(), op, ldo, workspace.data_ptr(),
        workspace.numel() * workspace.element_size()))
    return codes, norms, xhat


def rq4_quantize(x, rotors, centroids, bits, codes=None, norms=None, stream=None):
    """RotorQuant in the four-grade layout (4 codes per group, 172 at d = 128): (codes [n, W], norms [n])."""
    return rq_quantize(x, rotors, centroids, bits, codes, norms, stream, _fn="rq4_quantize", _cpg=4)


def rq4_dequantize(codes, norms, d, rotors, centroids, bits, out_dtype=None, xhat=None, stream=None):
    """Dequantize four-grade-layout codes [n, W] + norms [n] into x_hat [n, d]."""
    return rq_dequantize(codes, norms, d, rotors, centroids, bits, out_dtype, xhat, stream, _fn="rq4_dequantize")


def rq4_quantize_dequantize(x, rotors, centroids, bits, codes=None, norms=None, xhat=None, with_codes=True,
                            stream=None):
    """Fused roundtrip in the four-grade layout: (codes, norms, x_hat)."""
    return rq_quantize_dequantize(x, rotors, centroids, bits, codes, norms, xhat, with_codes, stream,
                                  _fn="rq4_quantize_dequantize", _cpg=4)


def device_status(stream=None):
    """Raise if a bounded device-side wait ran out since the last check (synchronises the stream)."""
    _lib.check("kvrq_device_status", lib().kvrq_device_status(_stream(stream)))


# ----------------------------------------------------------------------------- TurboQuant

def _tq_outputs(x_rows, d, cbits, device, codes, norms):
    torch = _torch()
    W = packed_words(d, cbits)
    if codes is None:
        codes = torch.empty((x_rows, W), dtype=torch.int32, device=device)
    if norms is None:
        norms = torch.empty((x_rows,), dtype=torch.float32, device=device)
    return codes, norms


def _pi_dtype(x_dtype):
    """Operand type of Pi for vectors of x_dtype: the same 16-bit type, fp16 for fp32 vectors."""
    torch = _torch()
    return torch.float16 if x_dtype == torch.float32 else x_dtype


def tq_workspace_bytes(rows, d):
    """Bytes of workspace the tiled prod path uses for `rows` rows (kvrq_tq_workspace_bytes)."""
    return int(lib().kvrq_tq_workspace_bytes(rows, d))


def tq_needs_workspace(d, dtype):
    """True when the prod calls at this d / vector dtype run on the tiled path and take a workspace."""
    torch = _torch()
    return d != 128 or dtype == torch.float32


def tq_workspace(n, d, device, max_bytes=256 << 20):
    """A workspace tensor for the prod calls: all n rows (rounded up to 128) if that fits in max_bytes,
    else the largest multiple of 128 rows that does (at least 128)."""
    torch = _torch()
    per_row = tq_workspace_bytes(1, d)
    rows = ((max(n, 1) + 127) // 128) * 128
    rows = max(128, min(rows, (max_bytes // per_row) // 128 * 128))
    return torch.empty((tq_workspace_bytes(rows, d),), dtype=torch.uint8, device=device)


def _ws_args(workspace, n, d, dtype, device):
    if not tq_needs_workspace(d, dtype):
        return None, 0, None
    if workspace is None:
        workspace = tq_workspace(n, d, device)
    return workspace.data_ptr(), workspace.numel() * workspace.element_size(), workspace


def tq_quantize_mse(x, pi, centroids, bits, codes=None, norms=None, stream=None):
    """TurboQuant-mse quantize rows of x [n, d]; pi [d, d] in x's dtype (fp16 for fp32 x).
    Returns (codes, norms)."""
    torch = _torch()
    n, d = x.shape
    codes, norms = _tq_outputs(n, d, bits, x.device, codes, norms)
    xp, ldx = _rows(x, "x")
    cp, ldc = _rows(codes, "codes")
    _lib.check("tq_quantize_mse", lib().tq_quantize_mse(_stream(stream), xp, _dtype_code(x), n, d, ldx,
                                                        _ptr(pi, "pi", _pi_dtype(x.dtype)),
                                                        _ptr(centroids, "centroids", torch.float32), bits, cp, ldc,
                                                        _ptr(norms, "norms", torch.float32)))
    return codes, norms


def tq_quantize_dequantize_mse(x, pi, centroids, bits, codes=None, norms=None, xhat=None, with_codes=True,
                               stream=None):
    """TurboQuant-mse roundtrip: returns (codes, norms, x_hat). Outside d = 128 with 16-bit vectors the
    codes and norms are always produced (the dequantize launch reads them)."""
    torch = _torch()
    n, d = x.shape
    if with_codes or tq_needs_workspace(d, x.dtype):
        codes, norms = _tq_outputs(n, d, bits, x.device, codes, norms)
    if xhat is None:
        xhat = torch.empty_like(x)
    xp, ldx = _rows(x, "x")
    cp, ldc = _rows(codes, "codes") if codes is not None else (None, packed_words(d, bits))
    op, ldo = _rows(xhat, "xhat")
    _lib.check("tq_quantize_dequantize_mse", lib().tq_quantize_dequantize_mse(
        _stream(stream), xp, _dtype_code(x), n, d, ldx, _ptr(pi, "pi", _pi_dtype(x.dtype)),
        _ptr(centroids, "centroids", torch.float32), bits, cp, ldc, _ptr(norms, "norms", torch.float32), op, ldo))
    return codes, norms, xhat


def tq_quantize_prod(x, pi, T, centroids, bits, codes=None, norms=None, signs=None, gammas=None, workspace=None,
                     stream=None):
    """TurboQuant-prod quantize (bits total: bits-1 mse bits + 1 QJL bit); T [m, d] fp16.
    `workspace` (uint8 device tensor, see tq_workspace) is allocated here when the tiled path needs one
    and none is given. Returns (codes, signs, gammas, norms)."""
    torch = _torch()
    n, d = x.shape
    m = T.shape[0]
    codes, norms = _tq_outputs(n, d, bits - 1, x.device, codes, norms)
    if signs is None:
        signs = torch.empty((n, m // 32), dtype=torch.int32, device=x.device)
    if gammas is None:
        gammas = torch.empty((n,), dtype=torch.float32, device=x.device)
    xp, ldx = _rows(x, "x")
    cp, ldc = _rows(codes, "codes")
    sp, lds = _rows(signs, "signs")
    wp, wbytes, _keep = _ws_args(workspace, n, d, x.dtype, x.device)
    _lib.check("tq_quantize_prod", lib().tq_quantize_prod(
        _stream(stream), xp, _dtype_code(x), n, d, ldx, _ptr(pi, "pi", _pi_dtype(x.dtype)),
        _ptr(T, "T", torch.float16), m, _ptr(centroids, "centroids", torch.float32), bits, cp, ldc, sp, lds,
        _ptr(gammas, "gammas", torch.float32), _ptr(norms, "norms", torch.float32), wp, wbytes))
    return codes, signs, gammas, norms


def tq_quantize_prod_noalloc(x, pi, T, centroids, bits, codes=None, norms=None, signs=None, gammas=None,
                             stream=None):
    """tq_quantize_prod through the library's static scratch instead of a workspace (the C call allocates
    nothing; outputs are allocated here when not given). Returns (codes, signs, gammas, norms)."""
    torch = _torch()
    n, d = x.shape
    m = T.shape[0]
    codes, norms = _tq_outputs(n, d, bits - 1, x.device, codes, norms)
    if signs is None:
        signs = torch.empty((n, m // 32), dtype=torch.int32, device=x.device)
    if gammas is None:
        gammas = torch.empty((n,), dtype=torch.float32, device=x.device)
    xp, ldx = _rows(x, "x")
    cp, ldc = _rows(codes, "codes")
    sp, lds = _rows(signs, "signs")
    _lib.check("tq_quantize_prod_noalloc", lib().tq_quantize_prod_noalloc(
        _stream(stream), xp, _dtype_code(x), n, d, ldx, _ptr(pi, "pi", _pi_dtype(x.dtype)),
        _ptr(T, "T", torch.float16), m, _ptr(centroids, "centroids", torch.float32), bits, cp, ldc, sp, lds,
        _ptr(gammas, "gammas", torch.float32), _ptr(norms, "norms", torch.float32)))
    return codes, signs, gammas, norms


def tq_dequantize(codes, norms, d, pi, centroids, bits, signs=None, gammas=None, T=None, xhat=None,
                  out_dtype=None, workspace=None, stream=None):
    """TurboQuant dequantize: mse when signs is None, prod otherwise (bits = total bits).
    The output dtype is out_dtype (default: pi's dtype; fp32 output takes an fp16 pi)."""
    torch = _torch()
    n = codes.shape[0]
    if xhat is None:
        xhat = torch.empty((n, d), dtype=out_dtype or pi.dtype, device=codes.device)
    m = T.shape[0] if T is not None else d
    cp, ldc = _rows(codes, "codes")
    sp, lds = _rows(signs, "signs") if signs is not None else (None, 0)
    op, ldo = _rows(xhat, "xhat")
    wp, wbytes, _keep = (None, 0, None) if signs is None else _ws_args(workspace, n, d, xhat.dtype, codes.device)
    _lib.check("tq_dequantize", lib().tq_dequantize(
        _stream(stream), cp, ldc, sp, lds, _ptr(gammas, "gammas", torch.float32), _ptr(norms, "norms", torch.float32),
        n, d, m, bits, _ptr(pi, "pi", _pi_dtype(xhat.dtype)), _ptr(T, "T", torch.float16),
        _ptr(centroids, "centroids", torch.float32), op, _dtype_code(xhat), ldo, wp, wbytes))
    return xhat


def qjl_sketch(r, T, signs=None, gammas=None, stream=None):
    """QJL sign sketch of the rows of r [n, d]: signs = sign(T r) packed (m/32 words per row), gammas = ||r||.
    T [m, d] in r's dtype (fp16 for fp32 r). Returns (signs, gammas)."""
    torch = _torch()
    n, d = r.shape
    m = T.shape[0]
    if signs is None:
        signs = torch.empty((n, m // 32), dtype=torch.int32, device=r.device)
    if gammas is None:
        gammas = torch.empty((n,), dtype=torch.float32, device=r.device)
    rp, ldr = _rows(r, "r")
    sp, lds = _rows(signs, "signs")
    _lib.check("qjl_sketch", lib().qjl_sketch(_stream(stream), rp, _dtype_code(r), n, d, ldr,
                                              _ptr(T, "T", _pi_dtype(r.dtype)), m, sp, lds,
                                              _ptr(gammas, "gammas", torch.float32), 1))
    return signs, gammas


# ----------------------------------------------------------------------------- scores

def kv_score_packed(method, q, codes, norms, bits, n_tokens, centroids, rotors=None, pi=None, T=None, signs=None,
                    gammas=None, scores=None, stream=None):
    """Scores from packed keys.

    q: [n_heads, group, d] CUDA tensor. codes: [n_heads, T_max, W] (int32 view of uint32),
    norms/gammas: [n_heads, T_max], signs: [n_heads, T_max, m/32]; the first n_tokens tokens
    of every head are scored. method: RQ_MSE, TQ_MSE or TQ_PROD; bits: the quantizer's total
    bits. Returns scores [n_heads, group, n_tokens] fp32."""
    torch = _torch()
    n_heads, group, d = q.shape
    if q.stride(2) != 1 or q.stride(1) != q.shape[2] or q.stride(0) != group * q.shape[2]:
        raise ValueError("q must be contiguous")
    if scores is None:
        scores = torch.empty((n_heads, group, n_tokens), dtype=torch.float32, device=q.device)
    m = T.shape[0] if T is not None else d
    def strides(t, name):
        if t is None:
            return None, 0, 0
        if not t.is_cuda or t.stride(-1) != 1:
            raise ValueError("%s must be a CUDA tensor with unit inner stride" % name)
        return t.data_ptr(), (t.stride(1) if t.dim() == 3 else 1), t.stride(0)
    cp, ldc, chs = strides(codes, "codes")
    sp, lds, shs = strides(signs, "signs")
    if norms.stride(-1) != 1 or (gammas is not None and gammas.stride() != norms.stride()):
        raise ValueError("norms/gammas must share one [n_heads, T_max] layout")
    pdt = _dtype_code(pi) if pi is not None else F16
    _lib.check("kv_score_packed", lib().kv_score_packed(
        _stream(stream), method, q.data_ptr(), _dtype_code(q), d, n_heads, group, d, bits, m, cp, ldc, chs, sp, lds,
        shs, _ptr(norms, "norms", torch.float32), _ptr(gammas, "gammas", torch.float32), norms.stride(0), n_tokens,
        _ptr(rotors, "rotors", torch.float32), _ptr(pi, "pi"), pdt, _ptr(T, "T", torch.float16),
        _ptr(centroids, "centroids", torch.float32), scores.data_ptr(), scores.stride(1)))
    return scores


def kv_cache_append(method, x, slot, bits, centroids, codes, norms, rotors=None, pi=None, T=None, signs=None,
                    gammas=None, stream=None):
    """Quantize x [rows, d] (one new vector per cache row) into slot `slot` of a packed cache:
    codes [rows, T_max, W], norms/gammas [rows, T_max], signs [rows, T_max, m/32]."""
    torch = _torch()
    rows, d = x.shape
    xp, ldx = _rows(x, "x")
    W = codes.shape[2]
    m = T.shape[0] if T is not None else d
    cp = codes.data_ptr() + slot * codes.stride(1) * 4
    sp = signs.data_ptr() + slot * signs.stride(1) * 4 if signs is not None else None
    np_ = norms.data_ptr() + slot * norms.stride(1) * 4
    gp = gammas.data_ptr() + slot * gammas.stride(1) * 4 if gammas is not None else None
    if gammas is not None and gammas.stride() != norms.stride():
        raise ValueError("norms and gammas must share one layout")
    _lib.check("kv_cache_append", lib().kv_cache_append(
        _stream(stream), method, xp, _dtype_code(x), rows, d, ldx, bits, _ptr(rotors, "rotors", torch.float32),
        _ptr(pi, "pi"), _ptr(T, "T", torch.float16), m, _ptr(centroids, "centroids", torch.float32), cp,
        codes.stride(0), sp, signs.stride(0) if signs is not None else 0, np_, gp, norms.stride(0)))


# ----------------------------------------------------------------------------- paged cache

def _paged(block_tables, seq_lens, page_tokens, n_seqs, kv_heads):
    torch = _torch()
    if block_tables.dtype != torch.int32 or seq_lens.dtype != torch.int32 or not block_tables.is_cuda:
        raise TypeError("block_tables and seq_lens must be int32 CUDA tensors")
    if block_tables.dim() != 2 or block_tables.stride(1) != 1 or not seq_lens.is_contiguous():
        raise ValueError("block_tables must be [n_seqs, ld_table] with unit inner stride")
    return _lib.KvrqPaged(block_tables.data_ptr(), block_tables.stride(0), seq_lens.data_ptr(), page_tokens, n_seqs,
                          kv_heads)


def _pool(t, name):
    """(pointer, row stride, pool-head stride) of a pool tensor [pool_heads, slots, W] (or [pool_heads, slots])."""
    if t is None:
        return None, 0, 0
    if not t.is_cuda or t.stride(-1) != 1:
        raise ValueError("%s must be a CUDA tensor with unit inner stride" % name)
    return t.data_ptr(), (t.stride(1) if t.dim() == 3 else 1), t.stride(0)


def kv_score_packed_paged(method, q, codes, norms, bits, block_tables, seq_lens, page_tokens, n_seqs, kv_heads,
                          max_tokens, centroids, rotors=None, pi=None, T=None, signs=None, gammas=None, scores=None,
                          stream=None):
    """Scores from a paged packed cache (kv_score_packed_paged in include/kvrq.h).

    q: [n_heads, group, d], head h = (layer * n_seqs + s) * kv_heads + k. Pools: codes [pool_heads, slots, W],
    norms/gammas [pool_heads, slots], signs [pool_heads, slots, m/32], pool head = layer * kv_heads + k.
    block_tables [n_seqs, ld_table] and seq_lens [n_seqs] int32 CUDA. Returns scores [n_heads, group,
    max_tokens] (entries t >= seq_lens[s] are left as they were)."""
    torch = _torch()
    n_heads, group, d = q.shape
    if not q.is_contiguous():
        raise ValueError("q must be contiguous")
    if scores is None:
        scores = torch.zeros((n_heads, group, max_tokens), dtype=torch.float32, device=q.device)
    m = T.shape[0] if T is not None else d
    cp, ldc, cps = _pool(codes, "codes")
    sp, lds, sps = _pool(signs, "signs")
    if norms.stride(-1) != 1 or (gammas is not None and gammas.stride() != norms.stride()):
        raise ValueError("norms/gammas must share one [pool_heads, slots] layout")
    pg = _paged(block_tables, seq_lens, page_tokens, n_seqs, kv_heads)
    pdt = _dtype_code(pi) if pi is not None else F16
    _lib.check("kv_score_packed_paged", lib().kv_score_packed_paged(
        _stream(stream), method, q.data_ptr(), _dtype_code(q), d, n_heads, group, d, bits, m, cp, ldc, cps, sp, lds,
        sps, _ptr(norms, "norms", torch.float32), _ptr(gammas, "gammas", torch.float32), norms.stride(0),
        ctypes.byref(pg), max_tokens, _ptr(rotors, "rotors", torch.float32), _ptr(pi, "pi"), pdt,
        _ptr(T, "T", torch.float16), _ptr(centroids, "centroids", torch.float32), scores.data_ptr(),
        scores.stride(1)))
    return scores


def kv_attention_packed_paged(k_method, q, k_codes, k_norms, k_bits, v_codes, v_norms, v_bits, block_tables,
                              seq_lens, page_tokens, n_seqs, kv_heads, max_tokens, k_centroids, v_rotors,
                              v_centroids, scale=None, k_rotors=None, pi=None, T=None, k_signs=None, k_gammas=None,
                              out=None, out_dtype=None, workspace=None, stream=None):
    """Decode attention over a paged packed cache (kv_attention_packed_paged in include/kvrq.h); pools and
    heads as kv_score_packed_paged, values v_codes [pool_heads, slots, Wv] and v_norms sharing the key norms'
    layout. Returns out [n_heads, group, d]."""
    torch = _torch()
    n_heads, group, d = q.shape
    if not q.is_contiguous():
        raise ValueError("q must be contiguous")
    if scale is None:
        scale = 1.0 / float(np.sqrt(d))
    if out is None:
        out = torch.empty((n_heads, group, d), dtype=out_dtype or torch.float32, device=q.device)
    m = T.shape[0] if T is not None else d
    need = attention_workspace_bytes(n_heads, group, max_tokens)
    if workspace is None:
        workspace = torch.empty((max(need, 16) + 15) // 16 * 4, dtype=torch.float32, device=q.device)
    kp, ldk, kps = _pool(k_codes, "k_codes")
    sp, lds, sps = _pool(k_signs, "k_signs")
    vp, ldv, vps = _pool(v_codes, "v_codes")
    if k_norms.stride(-1) != 1 or v_norms.stride() != k_norms.stride() or (
            k_gammas is not None and k_gammas.stride() != k_norms.stride()):
        raise ValueError("k_norms, k_gammas and v_norms must share one [pool_heads, slots] layout")
    pg = _paged(block_tables, seq_lens, page_tokens, n_seqs, kv_heads)
    pdt = _dtype_code(pi) if pi is not None else F16
    _lib.check("kv_attention_packed_paged", lib().kv_attention_packed_paged(
        _stream(stream), k_method, q.data_ptr(), _dtype_code(q), d, n_heads, group, d, float(scale), k_bits, m, kp,
        ldk, kps, sp, lds, sps, _ptr(k_norms, "k_norms", torch.float32), _ptr(k_gammas, "k_gammas", torch.float32),
        _ptr(k_rotors, "k_rotors", torch.float32), _ptr(pi, "pi"), pdt, _ptr(T, "T", torch.float16),
        _ptr(k_centroids, "k_centroids", torch.float32), vp, ldv, vps, _ptr(v_norms, "v_norms", torch.float32),
        v_bits, _ptr(v_rotors, "v_rotors", torch.float32), _ptr(v_centroids, "v_centroids", torch.float32),
        k_norms.stride(0), ctypes.byref(pg), max_tokens, out.data_ptr(), _dtype_code(out), out.stride(1),
        workspace.data_ptr(), workspace.numel() * workspace.element_size()))
    return out


def kv_cache_append_rows(method, x, dst_rows, bits, centroids, codes, norms, rotors=None, pi=None, T=None,
                         signs=None, gammas=None, stream=None):
    """Quantize row r of x [n, d] into pool row dst_rows[r] (int64 CUDA [n]) of flat pools: codes [rows, W],
    norms/gammas [rows], signs [rows, m/32] (e.g. a [pool_heads, slots, W] pool viewed as [pool_heads * slots,
    W], dst = pool_head * slots + slot)."""
    torch = _torch()
    n, d = x.shape
    if dst_rows.dtype != torch.int64 or not dst_rows.is_cuda or not dst_rows.is_contiguous():
        raise TypeError("dst_rows must be a contiguous int64 CUDA tensor")
    xp, ldx = _rows(x, "x")
    m = T.shape[0] if T is not None else d
    _lib.check("kv_cache_append_rows", lib().kv_cache_append_rows(
        _stream(stream), method, xp, _dtype_code(x), n, d, ldx, bits, _ptr(rotors, "rotors", torch.float32),
        _ptr(pi, "pi"), _ptr(T, "T", torch.float16), m, _ptr(centroids, "centroids", torch.float32),
        dst_rows.data_ptr(), codes.data_ptr(), codes.stride(0), signs.data_ptr() if signs is not None else None,
        signs.stride(0) if signs is not None else 0, norms.data_ptr(), gammas.data_ptr() if gammas is not None else None,
        norms.stride(0)))


def attention_workspace_bytes(n_heads, group, n_tokens):
    return int(lib().kvrq_attention_workspace_bytes(n_heads, group, n_tokens))


# ----------------------------------------------------------------------------- PolarQuant

PQ_WORDS = 16  # code words per d = 128 row: 496 bits of angle codes and fp16 radii


def pq_codebooks(level_bits=(4, 2, 2, 2)):
    """The [28] fp32 centroid table of pq_quantize_dequantize: the Lloyd-Max angle codebook of every level
    (pq_angle_codebook_init), level 1 first."""
    return np.concatenate([pq_angle_codebook_init(level, b)[0] for level, b in enumerate(level_bits, start=1)]
                          ).astype(np.float32)


def pq_quantize_dequantize(x, pi, centroids, codes=None, xhat=None, with_codes=True, stream=None):
    """PolarQuant fused roundtrip of rows x [n, 128] (fp16/bf16 CUDA): returns (codes [n, 16] int32 view of
    uint32, x_hat); codes is None when with_codes is False."""
    torch = _torch()
    n, d = x.shape
    if with_codes and codes is None:
        codes = torch.empty((n, PQ_WORDS), dtype=torch.int32, device=x.device)
    if xhat is None:
        xhat = torch.empty_like(x)
    xp, ldx = _rows(x, "x")
    cp, ldc = _rows(codes, "codes") if codes is not None else (None, PQ_WORDS)
    op, ldo = _rows(xhat, "xhat")
    _lib.check("pq_quantize_dequantize", lib().pq_quantize_dequantize(
        _stream(stream), xp, _dtype_code(x), n, d, ldx, _ptr(pi, "pi", pi.dtype),
        _ptr(centroids, "centroids", torch.float32), cp, ldc, op, ldo))
    return codes, xhat


def pq_dequantize(codes, d, pi, centroids, out_dtype=None, xhat=None, stream=None):
    """x_hat [n, d] from PolarQuant code rows [n, 16]."""
    torch = _torch()
    n = codes.shape[0]
    if xhat is None:
        xhat = torch.empty((n, d), dtype=out_dtype or pi.dtype, device=codes.device)
    cp, ldc = _rows(codes, "codes")
    op, ldo = _rows(xhat, "xhat")
    _lib.check("pq_dequantize", lib().pq_dequantize(_stream(stream), cp, ldc, n, d, _ptr(pi, "pi", pi.dtype),
                                                    _ptr(centroids, "centroids", torch.float32), op,
                                                    _dtype_code(xhat), ldo))
    return xhat


def attention_uses_tensor_cores(k_method, k_bits, v_bits, group):
    """True when kv_attention_packed runs both contractions on the tensor cores for this configuration
    (fp16 operands, outputs within 1e-2 of the row's largest |output|); False for the fp32 CUDA-core kernel."""
    return bool(lib().kvrq_attention_uses_tensor_cores(k_method, k_bits, v_bits, group))


def kv_attention_packed(k_method, q, k_codes, k_norms, k_bits, v_codes, v_norms, v_bits, n_tokens, k_centroids,
                        v_rotors, v_centroids, scale=None, k_rotors=None, pi=None, T=None, k_signs=None,
                        k_gammas=None, out=None, out_dtype=None, workspace=None, stream=None):
    """Decode attention from a packed KV cache.

    q: [n_heads, group, d] CUDA tensor. Keys as for kv_score_packed (k_codes [n_heads, T_max, Wk],
    k_norms/k_gammas [n_heads, T_max], k_signs [n_heads, T_max, m/32]); values RotorQuant codes
    v_codes [n_heads, T_max, Wv] with v_norms sharing the keys' norm layout. The first n_tokens
    tokens of every head are attended. scale defaults to 1/sqrt(d). Returns out [n_heads, group, d]
    (fp32 unless out_dtype is given)."""
    torch = _torch()
    n_heads, group, d = q.shape
    if q.stride(2) != 1 or q.stride(1) != d or q.stride(0) != group * d:
        raise ValueError("q must be contiguous")
    if scale is None:
        scale = 1.0 / float(np.sqrt(d))
    if out is None:
        out = torch.empty((n_heads, group, d), dtype=out_dtype or torch.float32, device=q.device)
    if out.stride(2) != 1 or out.stride(1) != out.shape[2] or out.stride(0) != group * out.shape[2]:
        raise ValueError("out must be contiguous")
    m = T.shape[0] if T is not None else d
    need = attention_workspace_bytes(n_heads, group, n_tokens)
    if workspace is None:
        workspace = torch.empty((max(need, 16) + 15) // 16 * 4, dtype=torch.float32, device=q.device)

    def strides(t, name):
        if t is None:
            return None, 0, 0
        if not t.is_cuda or t.stride(-1) != 1 or t.dim() != 3:
            raise ValueError("%s must be a 3-D CUDA tensor with unit inner stride" % name)
        return t.data_ptr(), t.stride(1), t.stride(0)

    kp, ldk, khs = strides(k_codes, "k_codes")
    sp, lds, shs = strides(k_signs, "k_signs")
    vp, ldv, vhs = strides(v_codes, "v_codes")
    if k_norms.stride(-1) != 1 or v_norms.stride() != k_norms.stride() or (
            k_gammas is not None and k_gammas.stride() != k_norms.stride()):
        raise ValueError("k_norms, k_gammas and v_norms must share one [n_heads, T_max] layout")
    pdt = _dtype_code(pi) if pi is not None else F16
    _lib.check("kv_attention_packed", lib().kv_attention_packed(
        _stream(stream), k_method, q.data_ptr(), _dtype_code(q), d, n_heads, group, d, float(scale), k_bits, m, kp,
        ldk, khs, sp, lds, shs, _ptr(k_norms, "k_norms", torch.float32), _ptr(k_gammas, "k_gammas", torch.float32),
        _ptr(k_rotors, "k_rotors", torch.float32), _ptr(pi, "pi"), pdt, _ptr(T, "T", torch.float16),
        _ptr(k_centroids, "k_centroids", torch.float32), vp, ldv, vhs, _ptr(v_norms, "v_norms", torch.float32),
        v_bits, _ptr(v_rotors, "v_rotors", torch.float32), _ptr(v_centroids, "v_centroids", torch.float32),
        k_norms.stride(0), n_tokens, out.data_ptr(), _dtype_code(out), d, _ptr(workspace, "workspace"),
        workspace.numel() * workspace.element_size()))
    return out


class PagedCache:
    """Host bookkeeping of a paged KV cache (kvrq_pages_* in include/kvrq.h): a pool of pages of
    page_tokens slots and per sequence its block table. Slots index the caller's packed device rows."""

    def __init__(self, n_pages, page_tokens):
        h = ctypes.c_void_p()
        _lib.check("kvrq_pages_create", lib().kvrq_pages_create(n_pages, page_tokens, ctypes.byref(h)))
        self._h = h
        self.page_tokens = page_tokens

    def close(self):
        h = getattr(self, "_h", None)
        self._h = None
        if h is not None and h.value and _lib is not None:
            _lib.load().kvrq_pages_destroy(h)

    def __del__(self):
        try:
            self.close()
        except Exception:  # interpreter shutdown: the library may already be gone
            pass

    def add_seq(self):
        sid = ctypes.c_int64(0)
        _lib.check("kvrq_pages_add_seq", lib().kvrq_pages_add_seq(self._h, ctypes.byref(sid)))
        return sid.value

    def append(self, seq, n_tokens):
        """Reserves n_tokens slots at the end of the sequence; returns the first new logical token."""
        first = ctypes.c_int64(0)
        _lib.check("kvrq_pages_append", lib().kvrq_pages_append(self._h, seq, n_tokens, ctypes.byref(first)))
        return first.value

    def slots(self, seq, first, count):
        out = np.zeros(count, dtype=np.int64)
        _lib.check("kvrq_pages_slots", lib().kvrq_pages_slots(self._h, seq, first, count,
                                                              out.ctypes.data_as(ctypes.c_void_p)))
        return out

    def block_table(self, seq):
        n_pages, n_tokens = ctypes.c_int64(0), ctypes.c_int64(0)
        lib().kvrq_pages_block_table(self._h, seq, None, 0, ctypes.byref(n_pages), ctypes.byref(n_tokens))
        out = np.zeros(n_pages.value, dtype=np.int32)
        _lib.check("kvrq_pages_block_table", lib().kvrq_pages_block_table(
            self._h, seq, out.ctypes.data_as(ctypes.c_void_p), len(out), ctypes.byref(n_pages),
            ctypes.byref(n_tokens)))
        return out, n_tokens.value

    def free_seq(self, seq):
        _lib.check("kvrq_pages_free_seq", lib().kvrq_pages_free_seq(self._h, seq))

    def stats(self):
        fp, ns = ctypes.c_int64(0), ctypes.c_int64(0)
        _lib.check("kvrq_pages_stats", lib().kvrq_pages_stats(self._h, ctypes.byref(fp), ctypes.byref(ns)))
        return fp.value, ns.value
