// Host-visible launch interface of the PolarQuant kernel.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "kvrq.h"

namespace kvrq {

enum PqMode { PQ_QDQ = 0, PQ_DQ = 1 };

constexpr int kPqWords = 16;       // code words per row at d = 128: 496 bits of codes and radii, 16 spare
constexpr int kPqCentroids = 28;   // 16 level-1 centroids, then 4 for each of levels 2, 3, 4

struct PqArgs {
  int64_t n;
  const float* centroids;    // [28] fp32
  uint32_t* codes_out;       // PQ_QDQ: [n][ldc] (may be NULL)
  const uint32_t* codes_in;  // PQ_DQ: [n][ldc]
  int64_t ldc;
  unsigned* status;
};

// map_x: rows of x (PQ_QDQ), map_pi: Pi [128][128], map_o: rows of x_hat; 64-column x 128-row
// boxes with 128-byte swizzle, all of the vector type dt (fp16 or bf16).
cudaError_t launch_pq(int mode, kvrq_dtype dt, const CUtensorMap& map_x, const CUtensorMap& map_pi,
                      const CUtensorMap& map_o, const PqArgs& a, cudaStream_t st, int num_sms);

}  // namespace kvrq
