// Host-visible launch interface of the TurboQuant tensor-core kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "kvrq.h"

namespace kvrq {

enum TqMode { TQ_MSE_Q = 0, TQ_MSE_QDQ = 1, TQ_PROD_Q = 2, TQ_DQ_MSE = 3, TQ_DQ_PROD = 4 };

// Arguments of one TurboQuant launch (device pointers; unused ones are NULL).
struct TqArgs {
  int64_t n;               // rows
  int d;                   // head dimension (= m, the QJL rows)
  const float* centroids;  // [2^bits] for the stored codes (b bits mse, b-1 bits prod)
  float qjl_scale;         // sqrt(pi/2) / m
  // quantize side
  int64_t ldx;
  uint32_t* codes_out;
  float* norms_out;
  uint32_t* signs_out;
  float* gammas_out;
  // dequantize side
  const uint32_t* codes_in;
  const float* norms_in;
  const uint32_t* signs_in;
  const float* gammas_in;
  int64_t ldc;  // code row stride (words)
  int64_t lds;  // sign row stride (words)
  int64_t ldn;  // norm and gamma row stride (floats)
  unsigned* status;
  const int64_t* out_rows;  // quantize, d = 128: row r's outputs go to row out_rows[r] (NULL: row r)
};

// map_x: input rows (quantize), map_pi: Pi [d][d], map_t: T [m][d] (fp16),
// map_o: x_hat rows (dequantize / roundtrip); all 64-column x 128-row boxes with
// 128-byte swizzle. `bits` is the stored code width.
cudaError_t launch_tq(int mode, kvrq_dtype dt, int bits, const CUtensorMap& map_x, const CUtensorMap& map_pi,
                      const CUtensorMap& map_t, const CUtensorMap& map_o, const TqArgs& a, cudaStream_t st,
                      int num_sms);

}  // namespace kvrq
