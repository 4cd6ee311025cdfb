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
};

// nb: MMA N (16, 32 or 64); cbits: stored code width.
cudaError_t launch_score(int method, int nb, int cbits, const ScoreArgs& a, cudaStream_t st);

}  // namespace kvrq
