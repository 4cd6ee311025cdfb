// Host-visible launch interface of the RotorQuant kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "kvrq.h"

namespace kvrq {

enum RqMode { RQ_Q = 0, RQ_DQ = 1, RQ_QDQ = 2 };

// Arguments of one RotorQuant launch (device pointers; unused ones are NULL).
struct RqArgs {
  int64_t n;  // rows
  int d;
  const float* rotors;     // [G][4]
  const float* centroids;  // [2^bits]
  // quantize side
  const void* x;
  int64_t ldx;
  uint32_t* codes_out;
  float* norms_out;
  // dequantize side
  const uint32_t* codes_in;
  const float* norms_in;
  void* xhat;
  int64_t ldo;
  int64_t ldc;  // row stride of codes (words), both directions
  int64_t ldn;  // row stride of norms (floats), both directions
  unsigned* status;  // device status word (bounded-wait time-outs)
  bool wide;         // any-d path: rows are streamed by bulk copy (rq_wide_smem_bytes > 0)
  int codes_per_group;  // 4: the four-grade layout (row kernel, d = 128); anything else: 3
  const int64_t* out_rows;  // quantize, d = 128: row r's outputs go to row out_rows[r] (NULL: row r)
};

// d = 128 thread-per-row kernel fed by TMA tensor maps over x and x_hat
// (128-byte boxes of 32 rows, 128-byte swizzle: one box per warp sub-tile).
cudaError_t launch_rq_row(int mode, kvrq_dtype dt, int bits, const CUtensorMap& map_x, const CUtensorMap& map_o,
                          const RqArgs& a, cudaStream_t st, int num_sms);

// Rows per box of the tensor maps launch_rq_row expects.
int rq_row_box_rows();
// Row dimensions (and types) the one-thread-per-row kernel takes: d = 128, and
// d = 256 for 16-bit rows.
bool rq_row_dims(int d, kvrq_dtype dt);

// Dynamic shared memory of the bulk-copy any-d kernel for d, or 0 when rows of
// d elements of elem_bytes cannot take it (row not a multiple of 16 bytes, a
// row over 16 KB, or tables and buffers over 227 KB).
int rq_wide_smem_bytes(int d, int bits, int elem_bytes);

// Any d / stride, warp-per-row kernel (a.wide selects the bulk-copy variant).
cudaError_t launch_rq_general(int mode, kvrq_dtype dt_in, kvrq_dtype dt_out, int bits, const RqArgs& a,
                              cudaStream_t st, int num_sms);

}  // namespace kvrq
