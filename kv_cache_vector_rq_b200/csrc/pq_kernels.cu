// PolarQuant at d = 128 on tcgen05 tensor cores ("TurboQuant и PolarQuant: математика
// квантизации KV-кэша в LLM": "Шаг 1: предобусловливание" (a fixed random rotation),
// "Полярное преобразование" (pairs of coordinates, then pairs of radii, become a radius
// and an angle, level after level), "Шаг 3: построение кодовых книг" (a Lloyd-Max codebook
// per level), "Степень сжатия" (four levels of 4, 2, 2, 2 bits and 8 radii of 16 bits:
// 496 bits per d = 128 vector)).
//
// Per row:
//   y = Pi x                                                   (tensor cores, fp32 in TMEM)
//   level 1: (a, b) = (y_2i, y_2i+1) -> angle in [0, 2 pi), radius sqrt(a^2 + b^2);
//   level l = 2, 3, 4: pairs of radii of level l-1 -> angle in [0, pi/2], radius;
//   angles -> nearest centroid of their level's codebook; the 8 level-4 radii -> fp16;
//   y_hat from the codes and the 16-bit radii (r cos c_hat, r sin c_hat, level by level),
//   x_hat = Pi^T y_hat                                         (tensor cores)
// No arctangent is evaluated. The level-1 codebook is the Lloyd-Max solution for the
// uniform angle, whose 16 boundaries are the multiples of pi/8: the code is the octant
// (from the signs of a and b and |b| against |a|) and the half of it (against tan(pi/8)
// or tan(3 pi/8)). A level-l angle (a, b >= 0) exceeds a boundary t exactly when
// b cos t > a sin t, so each of the three boundaries of a 2-bit code is one comparison of
// two products (a binary search: two comparisons per code).
//
// Layout of a row's 16 code words: words 0..7 the 64 level-1 codes (4 bits, LSB first),
// 8..9 the 32 level-2 codes, 10 the 16 level-3 codes, 11 the 8 level-4 codes (bits 0..15),
// 12..15 the 8 level-4 radii as fp16 pairs (radius 2c in the low half of word 12 + c).
//
// B200 shape (as the TurboQuant d = 128 kernel): a persistent CTA of 128 threads, one row
// per thread and TMEM lane; Pi resident in shared memory as 128-byte-swizzled tiles that
// are the MMA B operand K-major (y = x Pi^T) and MN-major (x_hat = y_hat Pi); the x tile
// arrives by TMA, y_hat is written back into it as the second A operand, and x_hat leaves
// from it by TMA. Two CTAs share an SM (256 TMEM columns each).

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include <type_traits>

#include "kvrq_device.cuh"
#include "pq_launch.h"

namespace kvrq {
namespace pq {

constexpr int kRows = 128;
constexpr int D = 128;
constexpr int kBoxBytes = kRows * 128;
constexpr int kTileBytes = 2 * kBoxBytes;
constexpr int W = kPqWords;

// shared constant table (fp32): [0, 16) cos of the level-1 centroids, [16, 32) their sines;
// level l = 2..4 at 32 + 14 (l - 2): [0, 3) cos of the three boundaries, [3, 6) their sines,
// [6, 10) cos of the four centroids, [10, 14) their sines
constexpr int kConsts = 32 + 3 * 14;

struct Smem {
  static constexpr int tile_off = 0;
  static constexpr int pi_off = kTileBytes;
  static constexpr int codes_off = pi_off + kTileBytes;  // [kRows][W]
  static constexpr int k_off = codes_off + kRows * W * 4;
  static constexpr int bar_off = ((k_off + kConsts * 4 + 7) / 8) * 8;  // x, params, mma
  static constexpr int tmem_off = bar_off + 3 * 8;
  static constexpr int bytes = tmem_off + 16;
  static constexpr int alloc = (bytes + 1024) < 80 * 1024 ? 80 * 1024 : bytes + 1024;  // <= 2 CTAs per SM
};

template <typename T>
struct IsBf16 {
  static constexpr bool value = std::is_same<T, __nv_bfloat16>::value;
};

// Level-1 code of (a, b): sector s of theta = atan2(b, a) in [0, 2 pi), cells [s pi/8, (s+1) pi/8)
// (ties to the lower code; a zero pair is sector 0, atan2(0, 0) = 0).
__device__ __forceinline__ uint32_t sector16(float a, float b, float t8, float t38) {
  uint32_t q;
  float x, y;  // the pair turned back by q quarter turns: x > 0, y >= 0 (or the zero pair)
  if (b >= 0.f) {
    if (a > 0.f || b == 0.f) {
      q = 0;
      x = a;
      y = b;
    } else {
      q = 1;
      x = b;
      y = -a;
    }
  } else {
    if (a < 0.f) {
      q = 2;
      x = -a;
      y = -b;
    } else {
      q = 3;
      x = -b;
      y = a;
    }
  }
  const uint32_t sub = (y > x * t8 ? 1u : 0u) + (y > x ? 1u : 0u) + (y > x * t38 ? 1u : 0u);
  return 4u * q + sub;
}

// 2-bit code of theta = atan2(b, a) (a, b >= 0) against boundaries t0 < t1 < t2, k = the
// level's table (cos t at k[0..3), sin t at k[3..6)); ties to the lower code
__device__ __forceinline__ uint32_t code4(float a, float b, const float* k) {
  const bool h1 = b * k[1] > a * k[4];
  return h1 ? 2u + (b * k[2] > a * k[5] ? 1u : 0u) : (b * k[0] > a * k[3] ? 1u : 0u);
}

// y_hat of the 32 coordinates of chunk c from the chunk's codes and radii (the inverse transform)
__device__ __forceinline__ void rebuild(const uint32_t* wc, int c, const float* s_k, float* yh) {
  const float* K2 = s_k + 32;
  const float* K3 = s_k + 46;
  const float* K4 = s_k + 60;
  const uint32_t rw = wc[12 + c];
  const float rh[2] = {__half2float(__ushort_as_half((unsigned short)(rw & 0xFFFFu))),
                       __half2float(__ushort_as_half((unsigned short)(rw >> 16)))};
  float q3[4], q2[8], q1[16];
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const uint32_t k = (wc[11] >> (4 * c + 2 * i)) & 3u;
    q3[2 * i] = rh[i] * K4[6 + k];
    q3[2 * i + 1] = rh[i] * K4[10 + k];
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t k = (wc[10] >> (8 * c + 2 * i)) & 3u;
    q2[2 * i] = q3[i] * K3[6 + k];
    q2[2 * i + 1] = q3[i] * K3[10 + k];
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint32_t k = (wc[8 + (c >> 1)] >> (16 * (c & 1) + 2 * i)) & 3u;
    q1[2 * i] = q2[i] * K2[6 + k];
    q1[2 * i + 1] = q2[i] * K2[10 + k];
  }
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const uint32_t k = (wc[2 * c + (i >> 3)] >> (4 * (i & 7))) & 15u;
    yh[2 * i] = q1[i] * s_k[k];
    yh[2 * i + 1] = q1[i] * s_k[16 + k];
  }
}

template <typename T, int MODE>
__global__ void __launch_bounds__(kRows, 1)
    pq_kernel(const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_pi,
              const __grid_constant__ CUtensorMap map_o, PqArgs a) {
  using SM = Smem;
  constexpr bool kQ = MODE == PQ_QDQ;
  constexpr uint32_t kNcols = 256;
  constexpr uint32_t kIdPi = umma_idesc_f16(IsBf16<T>::value, IsBf16<T>::value, false, D, kRows);  // X Pi^T
  constexpr uint32_t kIdPiT = umma_idesc_f16(IsBf16<T>::value, IsBf16<T>::value, true, D, kRows);  // Y Pi

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* s_tile = smem + SM::tile_off;
  uint8_t* s_pi = smem + SM::pi_off;
  uint32_t* s_codes = reinterpret_cast<uint32_t*>(smem + SM::codes_off);
  float* s_k = reinterpret_cast<float*>(smem + SM::k_off);
  uint64_t* bar_x = reinterpret_cast<uint64_t*>(smem + SM::bar_off);
  uint64_t* bar_p = bar_x + 1;
  uint64_t* bar_m = bar_x + 2;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + SM::tmem_off);

  const int tid = threadIdx.x, warp = tid >> 5;
  const int64_t n = a.n;
  const int64_t ntiles = (n + kRows - 1) / kRows;
  const uint32_t tile_s = smem_u32(s_tile), pi_s = smem_u32(s_pi);

  if (tid == 0) {
    if (kQ) tma_prefetch_desc(&map_x);
    tma_prefetch_desc(&map_pi);
    tma_prefetch_desc(&map_o);
    mbar_init(bar_x, 1);
    mbar_init(bar_p, 1);
    mbar_init(bar_m, 1);
    fence_barrier_init();
  }
  if (warp == 0) tmem_alloc(s_tmem, kNcols);
  // the constant table from the codebooks (boundaries: midpoints of neighbouring centroids)
  if (tid < 16) {
    const float c = a.centroids[tid];
    s_k[tid] = cosf(c);
    s_k[16 + tid] = sinf(c);
  } else if (tid < 16 + 3 * 7) {
    const int l = (tid - 16) / 7, j = (tid - 16) % 7;  // level l + 2; j < 3: boundary j, else centroid j - 3
    const float* c = a.centroids + 16 + 4 * l;
    float* k = s_k + 32 + 14 * l;
    if (j < 3) {
      const float t = 0.5f * (c[j] + c[j + 1]);
      k[j] = cosf(t);
      k[3 + j] = sinf(t);
    } else {
      k[6 + (j - 3)] = cosf(c[j - 3]);
      k[10 + (j - 3)] = sinf(c[j - 3]);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;
  const uint32_t tm_y = tmem, tm_2 = tmem + 128;
  const uint32_t lane_off = (uint32_t)(warp * 32) << 16;

  if (tid == 0) {
    mbar_arrive_expect_tx(bar_p, kTileBytes);
    for (int b = 0; b < 2; ++b) tma_load_2d(s_pi + b * kBoxBytes, &map_pi, b * 64, 0, bar_p);
  }
  bool ok = __syncthreads_and(mbar_wait(bar_p, 0, a.status));
  uint32_t par_x = 0, par_m = 0;

  auto mma = [&](uint32_t tm_d, uint32_t idesc, bool mn_b) {  // thread 0
    tc_fence_after();
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const uint32_t akoff = (uint32_t)((kk >> 2) * kBoxBytes + (kk & 3) * 32);
      const uint32_t bkoff = mn_b ? (uint32_t)(kk * 16 * 128) : akoff;
      umma_f16(tm_d, umma_desc_sw128(tile_s + akoff, 16, 1024),
               umma_desc_sw128(pi_s + bkoff, mn_b ? kBoxBytes : 16, 1024), idesc, kk > 0);
    }
    umma_commit(bar_m);
  };
  auto wait_mma = [&]() {
    const bool r = mbar_wait(bar_m, par_m, a.status);
    par_m ^= 1;
    tc_fence_after();
    return r;
  };
  auto put_chunk = [&](int j, const float* v) {
    *reinterpret_cast<uint4*>(s_tile + sw128_chunk(tid, j, kBoxBytes)) = Elem<T>::pack(v);
  };

  const float t8 = 0.41421356237309503f, t38 = 2.414213562373095f;  // tan(pi/8), tan(3 pi/8)
  for (int64_t tile = blockIdx.x; ok && tile < ntiles; tile += gridDim.x) {
    const int64_t row0 = tile * kRows;
    const int rows = (int)(n - row0 < (int64_t)kRows ? n - row0 : (int64_t)kRows);
    const int64_t row = row0 + tid;
    uint32_t wc[W];
    if constexpr (kQ) {
      if (tid == 0) {
        bulk_wait_read<0>();  // the previous x_hat store has left the tile buffer
        mbar_arrive_expect_tx(bar_x, kTileBytes);
        for (int b = 0; b < 2; ++b) tma_load_2d(s_tile + b * kBoxBytes, &map_x, b * 64, (int32_t)row0, bar_x);
      }
      ok = mbar_wait(bar_x, par_x, a.status);
      par_x ^= 1;
      if (!__syncthreads_and(ok)) break;
      if (tid == 0) mma(tm_y, kIdPi, false);  // y = Pi x per row
      if (!wait_mma()) ok = false;
#pragma unroll
      for (int w = 0; w < W; ++w) wc[w] = 0u;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        float y[32];
        tmem_ld32(tm_y + lane_off + 32 * c, y);
        // level 1: 16 pairs of coordinates
        float r1[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float a0 = y[2 * i], b0 = y[2 * i + 1];
          wc[2 * c + (i >> 3)] |= sector16(a0, b0, t8, t38) << (4 * (i & 7));
          r1[i] = sqrtf(fmaf(a0, a0, b0 * b0));
        }
        // levels 2..4: pairs of radii
        float r2[8], r3[4], r4[2];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          wc[8 + (c >> 1)] |= code4(r1[2 * i], r1[2 * i + 1], s_k + 32) << (16 * (c & 1) + 2 * i);
          r2[i] = sqrtf(fmaf(r1[2 * i], r1[2 * i], r1[2 * i + 1] * r1[2 * i + 1]));
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          wc[10] |= code4(r2[2 * i], r2[2 * i + 1], s_k + 46) << (8 * c + 2 * i);
          r3[i] = sqrtf(fmaf(r2[2 * i], r2[2 * i], r2[2 * i + 1] * r2[2 * i + 1]));
        }
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          wc[11] |= code4(r3[2 * i], r3[2 * i + 1], s_k + 60) << (4 * c + 2 * i);
          r4[i] = sqrtf(fmaf(r3[2 * i], r3[2 * i], r3[2 * i + 1] * r3[2 * i + 1]));
        }
        wc[12 + c] = (uint32_t)__half_as_ushort(__float2half_rn(r4[0])) |
                     ((uint32_t)__half_as_ushort(__float2half_rn(r4[1])) << 16);
      }
#pragma unroll
      for (int w = 0; w < W; ++w) s_codes[tid * W + w] = wc[w];
    } else {
      // the rows' code words (16 per row) from global memory
      for (int i = tid; i < rows * W; i += kRows) {
        const int r = i / W, w = i - r * W;
        s_codes[i] = __ldg(a.codes_in + (row0 + r) * a.ldc + w);
      }
      if (tid == 0) bulk_wait_read<0>();  // the previous x_hat store has left the tile buffer
      if (!__syncthreads_and(ok)) break;
#pragma unroll
      for (int w = 0; w < W; ++w) wc[w] = tid < rows ? s_codes[tid * W + w] : 0u;
    }
    // y_hat (the inverse transform of the codes and the 16-bit radii) as the second A operand
#pragma unroll
    for (int c = 0; c < D / 32; ++c) {
      float yh[32];
      rebuild(wc, c, s_k, yh);
#pragma unroll
      for (int q = 0; q < 4; ++q) put_chunk(4 * c + q, &yh[8 * q]);
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    if (tid == 0) mma(tm_2, kIdPiT, true);  // x_hat = Pi^T y_hat per row
    if (!wait_mma()) ok = false;
#pragma unroll
    for (int c = 0; c < D / 32; ++c) {
      float v[32];
      tmem_ld32(tm_2 + lane_off + 32 * c, v);
#pragma unroll
      for (int q = 0; q < 4; ++q) put_chunk(4 * c + q, &v[8 * q]);
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {
      for (int b = 0; b < 2; ++b) tma_store_2d(&map_o, b * 64, (int32_t)row0, s_tile + b * kBoxBytes);
      bulk_commit();
    }
    if (kQ && a.codes_out)
      for (int i = tid; i < rows * W; i += kRows) {
        const int r = i / W, w = i - r * W;
        a.codes_out[(row0 + r) * a.ldc + w] = s_codes[i];
      }
    (void)row;
    __syncthreads();  // the code words were read before the next tile overwrites them
  }
  if (tid == 0) bulk_wait_all<0>();
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kNcols);
  }
}

template <typename T, int MODE>
static cudaError_t launch_t(const CUtensorMap& mx, const CUtensorMap& mp, const CUtensorMap& mo, const PqArgs& a,
                            cudaStream_t st, int num_sms) {
  auto kern = pq_kernel<T, MODE>;
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Smem::alloc);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  const int64_t ntiles = (a.n + kRows - 1) / kRows;
  const int64_t grid = ntiles < (int64_t)num_sms * 2 ? ntiles : (int64_t)num_sms * 2;
  kern<<<(unsigned)grid, kRows, Smem::alloc, st>>>(mx, mp, mo, a);
  return cudaGetLastError();
}

}  // namespace pq

cudaError_t launch_pq(int mode, kvrq_dtype dt, const CUtensorMap& mx, const CUtensorMap& mp, const CUtensorMap& mo,
                      const PqArgs& a, cudaStream_t st, int num_sms) {
  if (dt == KVRQ_F16)
    return mode == PQ_QDQ ? pq::launch_t<__half, PQ_QDQ>(mx, mp, mo, a, st, num_sms)
                          : pq::launch_t<__half, PQ_DQ>(mx, mp, mo, a, st, num_sms);
  return mode == PQ_QDQ ? pq::launch_t<__nv_bfloat16, PQ_QDQ>(mx, mp, mo, a, st, num_sms)
                        : pq::launch_t<__nv_bfloat16, PQ_DQ>(mx, mp, mo, a, st, num_sms);
}

}  // namespace kvrq
