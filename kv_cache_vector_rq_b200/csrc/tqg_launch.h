// Host-visible launch interface of the tiled TurboQuant kernel (any head
// dimension that is a multiple of 128, fp32/fp16/bf16 vectors).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "kvrq.h"

namespace kvrq {

// One contraction D[rows][N] = A[rows][K] * B per launch, with the epilogue
// that the mode names:
//   G_MSE_Q     A = x, B = Pi (y = Pi x):          codes, norms
//   G_PROD_Q1   A = x, B = Pi:                      (b-1)-bit codes, norms, 2^8 r_rot (fp16) and
//                                                   per-tile sums of r_rot^2 into the workspace
//   G_PROD_Q2   A = 2^8 r_rot (workspace), B = T:   sign bits, gammas
//   G_SKETCH    A = r, B = T:                       sign bits, gammas = ||r||
//   G_DQ_MSE    A = c_hat (from codes), B = Pi^T:   x_hat = ||x|| Pi^T c_hat
//   G_DQ_PROD1  A = signs (+-1), B = T^T:           w = c_hat + sqrt(pi/2)/m gamma T^T s (workspace)
//   G_DQ_PROD2  A = w (workspace), B = Pi^T:        x_hat = ||x|| Pi^T w
enum TqgMode { G_MSE_Q = 0, G_PROD_Q1 = 1, G_PROD_Q2 = 2, G_SKETCH = 3, G_DQ_MSE = 4, G_DQ_PROD1 = 5, G_DQ_PROD2 = 6 };

struct TqgArgs {
  int64_t n;         // rows of this launch (local rows 0..n-1)
  int d;             // vector dimension
  int k_total;       // K of the contraction (multiple of 64)
  int n_total;       // N of the contraction (multiple of the N tile)
  int n_part;        // per-row partial sums written by G_PROD_Q1 (= d / its N tile)
  int64_t map_row0;  // row coordinate of local row 0 in the x / x_hat tensor maps
  const float* centroids;
  float qjl_scale;  // sqrt(pi/2) / m
  // fp32 vectors, read by the builder warps (x, r or the workspace w), local row 0
  const float* xf;
  int64_t ldx;
  // packed outputs / inputs, local row 0
  uint32_t* codes_out;
  const uint32_t* codes_in;
  int64_t ldc;
  uint32_t* signs_out;
  const uint32_t* signs_in;
  int64_t lds;
  float* norms_out;
  const float* norms_in;
  float* gammas_out;
  const float* gammas_in;
  int64_t ldn;
  // workspace: [rows][d] elements (2^8 r_rot in fp16, or w in the vector type),
  // then [rows][n_part] fp32 partial sums
  void* ws;
  float* part;
  unsigned* status;
};

// Tensor maps (128-byte swizzle): map_a = A rows (box 64 x 128 rows; unused when
// the builder warps write A), map_b = B (K-major: box 64 x N-tile rows; MN-major:
// box 64 x 64), map_o = x_hat rows (box 128 bytes x 128 rows).
// `n_tile` is 128 or 256; `bits` is the stored code width.
cudaError_t launch_tqg(int mode, kvrq_dtype dt, int bits, int n_tile, const CUtensorMap& map_a,
                       const CUtensorMap& map_b, const CUtensorMap& map_o, const TqgArgs& a, cudaStream_t st,
                       int num_sms);

// Shared-memory bytes the kernel needs (for validation / diagnostics).
int tqg_smem_bytes(int mode, kvrq_dtype dt, int n_tile);

}  // namespace kvrq
