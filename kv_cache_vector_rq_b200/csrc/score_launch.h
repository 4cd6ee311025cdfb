// Host-visible launch interface of the packed-code score kernel.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "kvrq.h"

namespace kvrq {

struct ScoreArgs {
  int64_t n_heads;          // KV heads (layers x batch x KV heads, flattened)
  int group;                // query heads per KV head
  int64_t n_tokens;
  int64_t tokens_per_cta;   // multiple of 128
  // queries [n_heads][group][ldq]
  const void* q;
  int64_t ldq;
  bool q_f32, q_bf16;
  // keys of head h, token t
  const uint32_t* codes;    // + h * codes_head_stride + t * ldc
  int64_t ldc, codes_head_stride;
  const uint32_t* signs;    // + h * signs_head_stride + t * lds (prod)
  int64_t lds, signs_head_stride;
  const float* norms;       // + h * tok_head_stride + t
  const float* gammas;      // prod
  int64_t tok_head_stride;
  // parameters
  const float* rotors;      // RotorQuant [43][4]
  const void* pi;           // TurboQuant [d][d], fp16 or bf16
  bool pi_bf16;
  const uint16_t* T;        // prod [m][d] fp16
  const float* centroids;   // stored-code codebook
  float qjl_scale;          // sqrt(pi/2) / m
  // scores [(h * group + g) * ld_scores + t]
  float* scores;
  int64_t ld_scores;
  unsigned* status;
  // paged cache (block_tables != NULL): head h = (layer * n_seqs + s) * kv_heads + k reads the rows of pool
  // head layer * kv_heads + k (the strides above then step pool heads), token t < seq_lens[s] at slot
  // page_tokens * block_tables[s * ld_table + t / page_tokens] + t % page_tokens
  const int32_t* block_tables;
  int64_t ld_table;
  const int32_t* seq_lens;
  int page_tokens;
  int n_seqs;
  int kv_heads;
  // polls of the tile and MMA waits of the main loop before they give up (negative: the default;
  // 0: they give up at once); the waits that drain copies and MMAs in flight always use the default
  int32_t spin_limit;
};

// Pool head, block-table row and token count of head `head` of a paged call, or of a contiguous one
// (head itself, no table, n_tokens).
struct PagedHead {
  int64_t pool_head;
  const int32_t* table;
  int64_t n_tokens;
  int shift;   // log2(page_tokens) when it is a power of two, else -1
  int ptok;
  __device__ __forceinline__ int64_t slot(int64_t t) const {
    if (!table) return t;
    if (shift >= 0) return ((int64_t)__ldg(table + (t >> shift)) << shift) + (t & (ptok - 1));
    return (int64_t)__ldg(table + t / ptok) * ptok + t % ptok;
  }
};

__device__ __forceinline__ PagedHead paged_head(int64_t head, int64_t n_tokens, const int32_t* tables, int64_t ld_table,
                                                const int32_t* seq_lens, int page_tokens, int n_seqs, int kv_heads) {
  PagedHead p;
  p.pool_head = head;
  p.table = nullptr;
  p.n_tokens = n_tokens;
  p.ptok = page_tokens;
  p.shift = -1;
  if (tables) {
    const int64_t k = head % kv_heads, s = (head / kv_heads) % n_seqs, layer = head / ((int64_t)kv_heads * n_seqs);
    p.pool_head = layer * kv_heads + k;
    p.table = tables + s * ld_table;
    const int64_t len = __ldg(seq_lens + s);
    p.n_tokens = len < n_tokens ? (len > 0 ? len : 0) : n_tokens;
    if ((page_tokens & (page_tokens - 1)) == 0) p.shift = __ffs(page_tokens) - 1;
  }
  return p;
}

// nb: MMA N (16, 32 or 64); cbits: stored code width.
cudaError_t launch_score(int method, int nb, int cbits, const ScoreArgs& a, cudaStream_t st);

}  // namespace kvrq
