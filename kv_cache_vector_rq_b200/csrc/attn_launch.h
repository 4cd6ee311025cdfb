// Host-visible launch interface of the decode-attention kernels.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "kvrq.h"

namespace kvrq {

constexpr int kAttnQS = 132;   // floats per rotated-query row (3G = 129 used for RotorQuant keys, d = 128 for TurboQuant)
constexpr int kAttnAS = 132;   // floats per value-accumulator row (3G = 129 rotated value coordinates used)
constexpr int kAttnSub = 256;  // tokens per sub-chunk: one per thread of the chunk kernel
constexpr int kAttnMaxChunks = 1024;
constexpr int kAttnTcParts = 3;  // tensor-core path: decode warpgroups per CTA, each taking its own work items

struct AttnArgs {
  int64_t n_heads;          // KV heads (layers x batch x KV heads, flattened)
  int group;                // query heads per KV head
  int64_t n_tokens;
  int64_t tokens_per_cta;   // multiple of kAttnSub
  int n_chunks;             // ceil(n_tokens / tokens_per_cta)
  // queries [n_heads][group][ldq]
  const void* q;
  int64_t ldq;
  bool q_f32, q_bf16;
  float scale;              // logit scale
  // keys of head h, token t
  const uint32_t* k_codes;  // + h * k_head_stride + t * ldk
  int64_t ldk, k_head_stride;
  const uint32_t* k_signs;  // + h * s_head_stride + t * lds (prod)
  int64_t lds, s_head_stride;
  const float* k_norms;     // + h * tok_head_stride + t
  const float* k_gammas;    // prod
  const float* k_rotors;    // RotorQuant keys [43][4]
  const void* pi;           // TurboQuant keys [d][d], fp16 or bf16
  bool pi_bf16;
  const uint16_t* T;        // prod [m][d] fp16
  const float* k_centroids; // stored key-code codebook
  float qjl_scale;          // sqrt(pi/2) / m
  // RotorQuant values of head h, token t
  const uint32_t* v_codes;  // + h * v_head_stride + t * ldv
  int64_t ldv, v_head_stride;
  const float* v_norms;     // + h * tok_head_stride + t
  const float* v_rotors;    // [43][4]
  const float* v_centroids;
  int v_bits;
  int64_t tok_head_stride;
  // outputs [(h * group + g) * ldo + i], i < d
  void* out;
  int64_t ldo;
  int odtype;               // kvrq_dtype
  // workspace (caller-owned), rows = n_heads * group
  float* ws_q;              // [rows][kAttnQS] rotated queries
  float* ws_sq;             // [rows][128]     T q' (prod)
  float* ws_acc;            // [rows][n_chunks][kAttnAS] per-chunk value sums, rotated domain
  float* ws_ml;             // [rows][n_chunks][2] per-chunk (max logit, sum of weights)
  unsigned* status;         // device status word (bounded-wait time-outs of the tensor-core path)
  int32_t spin_limit;       // polls of the tensor-core path's tile-copy waits (< 0: the default)
  // paged cache (block_tables != NULL, tensor-core path): as ScoreArgs; the head strides then step pool heads
  const int32_t* block_tables;
  int64_t ld_table;
  const int32_t* seq_lens;
  int page_tokens;
  int n_seqs;
  int kv_heads;
};

// Tokens per chunk CTA of the CUDA-core path (a multiple of kAttnSub), tokens per
// work item of the tensor-core path (a multiple of 128), and the workspace the call
// needs (enough for either path); all depend on the sizes only, not on the device.
int64_t attn_tokens_per_cta(int64_t n_heads, int64_t n_tokens);
int64_t attn_tc_tokens_per_item(int64_t n_heads, int64_t n_tokens);
size_t attn_workspace_bytes(int64_t n_heads, int group, int64_t n_tokens);

// Whether the tensor-core kernel takes keys of k_method with k_cbits-bit stored codes,
// values of v_bits bits and `group` query rows per KV head.
bool attn_tc_supported(int k_method, int k_cbits, int v_bits, int group);

// The tensor-core chunk kernel (a.tokens_per_cta = tokens per work item, a.n_chunks =
// work items per head, one partial each); persistent, at most num_sms CTAs.
cudaError_t launch_attention_tc(int k_method, int k_cbits, const AttnArgs& a, cudaStream_t st, int num_sms);

// k_method: kvrq_method of the keys; k_cbits: stored key-code width. Chooses the path
// and sets a.tokens_per_cta and a.n_chunks for it.
cudaError_t launch_attention(int k_method, int k_cbits, AttnArgs a, cudaStream_t st, int num_sms);

}  // namespace kvrq
