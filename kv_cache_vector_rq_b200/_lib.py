"""ctypes declarations of libkvrq.so (the C ABI in include/kvrq.h).

Loading fails loudly when the shared library has not been built: there is no
fallback implementation.
"""

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libkvrq.so")

c_int, c_i64, c_u64, c_f64 = ctypes.c_int, ctypes.c_int64, ctypes.c_uint64, ctypes.c_double
c_vp = ctypes.c_void_p
c_dp = ctypes.POINTER(ctypes.c_double)
c_ip = ctypes.POINTER(ctypes.c_int)

# name -> (restype, argtypes); one entry per function in include/kvrq.h
SIGNATURES = {
    "kvrq_version": (ctypes.c_char_p, []),
    "kvrq_last_error_string": (ctypes.c_char_p, []),
    "kvrq_device_status": (c_int, [c_vp]),
    "kvrq_packed_words": (c_i64, [c_i64, c_int]),
    "kvrq_rq_groups": (c_int, [c_int]),
    "tq_codebook_init": (c_int, [c_int, c_int, c_f64, c_int, c_dp, c_dp, c_ip]),
    "pq_angle_codebook_init": (c_int, [c_int, c_int, c_f64, c_int, c_dp, c_dp, c_ip]),
    "rq_rotors_init": (c_int, [c_int, c_u64, c_dp]),
    "tq_rotation_init": (c_int, [c_int, c_u64, c_dp]),
    "qjl_matrix_init": (c_int, [c_int, c_int, c_u64, c_dp]),
    "kvrq_normals": (c_int, [c_u64, c_i64, c_i64, c_dp]),
    # stream, x, xdtype, n, d, ldx, rotors, centroids, bits, codes, ldc, norms
    "rq_quantize": (c_int, [c_vp, c_vp, c_int, c_i64, c_int, c_i64, c_vp, c_vp, c_int, c_vp, c_i64, c_vp]),
    # stream, codes, ldc, norms, n, d, rotors, centroids, bits, xhat, odtype, ldo
    "rq_dequantize": (c_int, [c_vp, c_vp, c_i64, c_vp, c_i64, c_int, c_vp, c_vp, c_int, c_vp, c_int, c_i64]),
    # stream, x, xdtype, n, d, ldx, rotors, centroids, bits, codes, ldc, norms, xhat, ldo
    "rq_quantize_dequantize": (c_int, [c_vp, c_vp, c_int, c_i64, c_int, c_i64, c_vp, c_vp, c_int, c_vp, c_i64, c_vp,
                                       c_vp, c_i64]),
    # stream, x (host), xdtype, n, d, ldx, rotors, centroids, bits, codes (host), ldc, norms (host), xhat (host),
    # ldo, workspace (device), workspace bytes
    "rq_quantize_dequantize_host": (c_int, [c_vp, c_vp, c_int, c_i64, c_int, c_i64, c_vp, c_vp, c_int, c_vp, c_i64,
                                            c_vp, c_vp, c_i64, c_vp, ctypes.c_size_t]),
    "kvrq_host_workspace_bytes": (ctypes.c_size_t, [c_int, c_int, c_int, c_i64]),
    "rq4_quantize": (c_int, [c_vp, c_vp, c_int, c_i64, c_int, c_i64, c_vp, c_vp, c_int, c_vp, c_i64, c_vp]),
    "rq4_dequantize": (c_int, [c_vp, c_vp, c_i64, c_vp, c_i64, c_int, c_vp, c_vp, c_int, c_vp, c_int, c_i64]),
    "rq4_quantize_dequantize": (c_int, [c_vp, c_vp, c_int, c_i64, c_int, c_i64, c_vp, c_vp, c_int, c_vp, c_i64, c_vp,
                                        c_vp, c_i64]),
    # stream, x, xdtype, n, d, ldx, pi, centroids, bits, codes, ldc, norms
    "tq_quantize_mse": (c_int, [c_vp, c_vp, c_int, c_i64, c_int, c_i64, c_vp, c_vp, c_int, c_vp, c_i64, c_vp]),
    # ... + xhat, ldo
    "tq_quantize_dequantize_mse": (c_int, [c_vp, c_vp, c_int, c_i64, c_int, c_i64, c_vp, c_vp, c_int, c_vp, c_i64,
                                           c_vp, c_vp, c_i64]),
    # rows, d
    "kvrq_tq_workspace_bytes": (ctypes.c_size_t, [c_i64, c_int]),
    # stream, x, xdtype, n, d, ldx, pi, T, m, centroids, bits, codes, ldc, signs, lds, gammas, norms, workspace,
    # workspace_bytes
    "tq_quantize_prod": (c_int, [c_vp, c_vp, c_int, c_i64, c_int, c_i64, c_vp, c_vp, c_int, c_vp, c_int, c_vp, c_i64,
                                 c_vp, c_i64, c_vp, c_vp, c_vp, ctypes.c_size_t]),
    # stream, x, xdtype, n, d, ldx, pi, T, m, centroids, bits, codes, ldc, signs, lds, gammas, norms
    "tq_quantize_prod_noalloc": (c_int, [c_vp, c_vp, c_int, c_i64, c_int, c_i64, c_vp, c_vp, c_int, c_vp, c_int, c_vp,
                                         c_i64, c_vp, c_i64, c_vp, c_vp]),
    # stream, codes, ldc, signs, lds, gammas, norms, n, d, m, bits, pi, T, centroids, xhat, odtype, ldo, workspace,
    # workspace_bytes
    "tq_dequantize": (c_int, [c_vp, c_vp, c_i64, c_vp, c_i64, c_vp, c_vp, c_i64, c_int, c_int, c_int, c_vp, c_vp,
                              c_vp, c_vp, c_int, c_i64, c_vp, ctypes.c_size_t]),
    # stream, r, rdtype, n, d, ldr, T, m, signs, lds, gammas, ldn
    "qjl_sketch": (c_int, [c_vp, c_vp, c_int, c_i64, c_int, c_i64, c_vp, c_int, c_vp, c_i64, c_vp, c_i64]),
    # stream, method, q, qdtype, ldq, n_heads, group, d, bits, m, codes, ldc, codes_head_stride, signs, lds,
    # signs_head_stride, norms, gammas, tok_head_stride, n_tokens, rotors, pi, pi_dtype, T, centroids, scores,
    # ld_scores
    "kv_score_packed": (c_int, [c_vp, c_int, c_vp, c_int, c_i64, c_i64, c_int, c_int, c_int, c_int, c_vp, c_i64,
                                c_i64, c_vp, c_i64, c_i64, c_vp, c_vp, c_i64, c_i64, c_vp, c_vp, c_int, c_vp, c_vp,
                                c_vp, c_i64]),
    # stream, method, x, xdtype, n_rows, d, ldx, bits, rotors, pi, T, m, centroids, codes, codes_row_stride,
    # signs, signs_row_stride, norms, gammas, norm_row_stride
    "kv_cache_append": (c_int, [c_vp, c_int, c_vp, c_int, c_i64, c_int, c_i64, c_int, c_vp, c_vp, c_vp, c_int, c_vp,
                                c_vp, c_i64, c_vp, c_i64, c_vp, c_vp, c_i64]),
    # n_heads, group, n_tokens
    "kvrq_attention_workspace_bytes": (ctypes.c_size_t, [c_i64, c_int, c_i64]),
    # stream, k_method, q, qdtype, ldq, n_heads, group, d, scale, k_bits, m, k_codes, ldk, k_head_stride, k_signs,
    # lds, s_head_stride, k_norms, k_gammas, k_rotors, pi, pi_dtype, T, k_centroids, v_codes, ldv, v_head_stride,
    # v_norms, v_bits, v_rotors, v_centroids, tok_head_stride, n_tokens, out, odtype, ldo, workspace, workspace_bytes
    "kv_attention_packed": (c_int, [c_vp, c_int, c_vp, c_int, c_i64, c_i64, c_int, c_int, ctypes.c_float, c_int, c_int,
                                    c_vp, c_i64, c_i64, c_vp, c_i64, c_i64, c_vp, c_vp, c_vp, c_vp, c_int, c_vp, c_vp,
                                    c_vp, c_i64, c_i64, c_vp, c_int, c_vp, c_vp, c_i64, c_i64, c_vp, c_int, c_i64, c_vp,
                                    ctypes.c_size_t]),
    # stream, x, xdtype, n, d, ldx, pi, centroids, codes, ldc, xhat, ldo
    "pq_quantize_dequantize": (c_int, [c_vp, c_vp, c_int, c_i64, c_int, c_i64, c_vp, c_vp, c_vp, c_i64, c_vp, c_i64]),
    # stream, codes, ldc, n, d, pi, centroids, xhat, odtype, ldo
    "pq_dequantize": (c_int, [c_vp, c_vp, c_i64, c_i64, c_int, c_vp, c_vp, c_vp, c_int, c_i64]),
    # stream, method, q, qdtype, ldq, n_heads, group, d, bits, m, codes, ldc, codes_pool_stride, signs, lds,
    # signs_pool_stride, norms, gammas, tok_pool_stride, paged, max_tokens, rotors, pi, pi_dtype, T, centroids,
    # scores, ld_scores
    "kv_score_packed_paged": (c_int, [c_vp, c_int, c_vp, c_int, c_i64, c_i64, c_int, c_int, c_int, c_int, c_vp,
                                      c_i64, c_i64, c_vp, c_i64, c_i64, c_vp, c_vp, c_i64, c_vp, c_i64, c_vp, c_vp,
                                      c_int, c_vp, c_vp, c_vp, c_i64]),
    # as kv_attention_packed with pool strides, then paged, max_tokens before out
    "kv_attention_packed_paged": (c_int, [c_vp, c_int, c_vp, c_int, c_i64, c_i64, c_int, c_int, ctypes.c_float,
                                          c_int, c_int, c_vp, c_i64, c_i64, c_vp, c_i64, c_i64, c_vp, c_vp, c_vp,
                                          c_vp, c_int, c_vp, c_vp, c_vp, c_i64, c_i64, c_vp, c_int, c_vp, c_vp,
                                          c_i64, c_vp, c_i64, c_vp, c_int, c_i64, c_vp, ctypes.c_size_t]),
    # stream, method, x, xdtype, n_rows, d, ldx, bits, rotors, pi, T, m, centroids, dst_rows, codes, ldc, signs,
    # lds, norms, gammas, ldn
    "kv_cache_append_rows": (c_int, [c_vp, c_int, c_vp, c_int, c_i64, c_int, c_i64, c_int, c_vp, c_vp, c_vp, c_int,
                                     c_vp, c_vp, c_vp, c_i64, c_vp, c_i64, c_vp, c_vp, c_i64]),
    "kvrq_test_fail_allocations": (None, [c_int]),
    "kvrq_set_wait_limit": (None, [c_i64]),
    "kvrq_params_export": (c_int, [ctypes.c_char_p, c_int, c_int, c_int, ctypes.c_uint64]),
    "kvrq_params_import": (c_int, [ctypes.c_char_p, c_int, c_int, c_int, ctypes.POINTER(ctypes.c_uint64), c_vp, c_vp,
                                   c_vp, c_vp]),
    "kvrq_attention_uses_tensor_cores": (c_int, [c_int, c_int, c_int, c_int]),
    "kvrq_pages_create": (c_int, [c_i64, c_int, ctypes.POINTER(c_vp)]),
    "kvrq_pages_destroy": (None, [c_vp]),
    "kvrq_pages_add_seq": (c_int, [c_vp, ctypes.POINTER(c_i64)]),
    "kvrq_pages_append": (c_int, [c_vp, c_i64, c_i64, ctypes.POINTER(c_i64)]),
    "kvrq_pages_slots": (c_int, [c_vp, c_i64, c_i64, c_i64, c_vp]),
    "kvrq_pages_block_table": (c_int, [c_vp, c_i64, c_vp, c_i64, ctypes.POINTER(c_i64), ctypes.POINTER(c_i64)]),
    "kvrq_pages_free_seq": (c_int, [c_vp, c_i64]),
    "kvrq_pages_stats": (c_int, [c_vp, ctypes.POINTER(c_i64), ctypes.POINTER(c_i64)]),
}

_lib = None


class KvrqError(RuntimeError):
    """A non-OK status from the library."""

    def __init__(self, name, status, message):
        super().__init__("%s failed with status %d: %s" % (name, status, message))
        self.status = status


def load():
    """Load libkvrq.so (once) and declare every function's signature."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError("libkvrq.so is not built (expected at %s); run __graft_entry__.build()" % LIB_PATH)
    lib = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def check(name, status):
    if status != 0:
        msg = load().kvrq_last_error_string().decode()
        raise KvrqError(name, status, msg)


class KvrqPaged(ctypes.Structure):
    """struct kvrq_paged of include/kvrq.h."""
    _fields_ = [("block_tables", ctypes.c_void_p), ("ld_table", ctypes.c_int64), ("seq_lens", ctypes.c_void_p),
                ("page_tokens", ctypes.c_int32), ("n_seqs", ctypes.c_int32), ("kv_heads", ctypes.c_int32)]
