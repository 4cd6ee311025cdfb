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
// No arctangent and, below the last level, no square root is evaluated. The level-1 codebook
// is the Lloyd-Max solution for the uniform angle, whose 16 boundaries are the multiples of
// pi/8: with phi = atan(|b| / |a|) in [0, pi/2], n = the number of the boundaries pi/8, pi/4,
// 3 pi/8 that phi exceeds (|b| against |a| tan(pi/8), |a|, |a| tan(3 pi/8)); the code is n in
// the first quadrant, 7 - n in the second, 8 + n in the third and 15 - n in the fourth, which is
// n XOR (8 [b < 0] + 7 [sign a != sign b]). A level-l angle (l >= 2) of the radii
// (sqrt A, sqrt B) exceeds a boundary t exactly when B > A tan^2 t, so levels 2..4 work on the
// squared radii A (sums of squares of 2^l coordinates) and only the 8 stored radii take a
// square root.
//
// Layout of a row's 16 code words: words 0..7 the 64 level-1 codes (4 bits, LSB first),
// 8..9 the 32 level-2 codes, 10 the 16 level-3 codes, 11 the 8 level-4 codes (bits 0..15),
// 12..15 the 8 level-4 radii as fp16 pairs (radius 2c in the low half of word 12 + c).
// Every level-4 radius covers 16 coordinates, so the transform of a row splits into independent
// 32-column chunks: chunk c gives words 2c, 2c + 1, bits 16 (c & 1) .. of word 8 + c / 2,
// bits 8c .. of word 10, bits 4c .. of word 11 and word 12 + c.
//
// B200 shape: a persistent CTA of 256 threads works on 128-row tiles, two threads per row
// (TMEM lane): warp w takes lanes 32 (w & 3) .. and half h = w / 4 of the columns (chunks 2h,
// 2h + 1). Pi is resident in shared memory as 128-byte-swizzled tiles that are the MMA B
// operand K-major (y = x Pi^T) and MN-major (x_hat = y_hat Pi). Two tile buffers alternate: the
// TMA load of the next tile's x is issued as soon as this tile's first product has read its
// own, and lands while this tile is transformed; y_hat is written over x as the second A
// operand, x_hat over y_hat, and leaves by TMA. Code words go from registers to global memory
// (the second half's bits of words 10 and 11 pass through shared memory). Two CTAs share an SM
// (256 TMEM columns each: y and x_hat accumulators).

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
constexpr int kThreads = 256;
constexpr int kBoxBytes = kRows * 128;
constexpr int kTileBytes = 2 * kBoxBytes;

struct Smem {
  static constexpr int buf_off = 0;                     // two tiles: x, then y_hat, then x_hat
  static constexpr int pi_off = 2 * kTileBytes;
  static constexpr int cs_off = pi_off + kTileBytes;    // float2 [28]: (cos, sin) of every centroid
  static constexpr int tan_off = cs_off + kPqCentroids * 8;  // float [9]: tan^2 of the level 2..4 boundaries
  static constexpr int xchg_off = tan_off + 12 * 4;     // u32 [kRows]: half 1's bits of words 10 and 11
  static constexpr int bar_off = xchg_off + kRows * 4;  // x[2], params, mma
  static constexpr int tmem_off = bar_off + 4 * 8;
  static constexpr int bytes = tmem_off + 16;
  static constexpr int alloc = bytes + 1024;
};
static_assert(2 * (Smem::alloc + 1024) <= 228 * 1024, "two CTAs per SM");

template <typename T>
struct IsBf16 {
  static constexpr bool value = std::is_same<T, __nv_bfloat16>::value;
};

// all-ones if x > y (x < y), else 0
__device__ __forceinline__ uint32_t set_gt(float x, float y) {
  uint32_t r;
  asm("set.gt.u32.f32 %0, %1, %2;" : "=r"(r) : "f"(x), "f"(y));
  return r;
}
__device__ __forceinline__ uint32_t set_lt(float x, float y) {
  uint32_t r;
  asm("set.lt.u32.f32 %0, %1, %2;" : "=r"(r) : "f"(x), "f"(y));
  return r;
}

// Level-1 code of (a, b): the cell of theta = atan2(b, a) in [0, 2 pi) among the 16 of width
// pi/8; a boundary angle takes either neighbouring code, a zero pair (of either sign) code 0.
__device__ __forceinline__ uint32_t sector16(float a, float b) {
  constexpr float t8 = 0.41421356237309503f, t38 = 2.414213562373095f;  // tan(pi/8), tan(3 pi/8)
  const float fa = fabsf(a), fb = fabsf(b);
  const uint32_t n = 0u - (set_gt(fb, fa * t8) + set_gt(fb, fa) + set_gt(fb, fa * t38));
  const uint32_t mb = set_lt(b, 0.f), ma = set_lt(a, 0.f);
  return n ^ ((mb & 8u) | ((ma ^ mb) & 7u));
}

// 2-bit code of the angle of the radii (sqrt A, sqrt B) against boundaries with tan^2 = T[0..3)
// (ties to the lower code)
__device__ __forceinline__ uint32_t code4(float A, float B, const float* T) {
  return 0u - (set_gt(B, A * T[0]) + set_gt(B, A * T[1]) + set_gt(B, A * T[2]));
}

// The code words of one thread's half row (chunks 2h, 2h + 1).
struct Half {
  uint32_t l1[4];  // words 4h .. 4h + 3
  uint32_t l2;     // word 8 + h
  uint32_t l3;     // bits 16h .. 16h + 15 of word 10, shifted down
  uint32_t l4;     // bits 8h .. 8h + 7 of word 11, shifted down
  uint32_t r[2];   // words 12 + 2h, 13 + 2h
};

// Quantize chunk cc (0, 1) of the half from its 32 fp32 coordinates.
__device__ __forceinline__ void quantize_chunk(const float* y, int cc, const float* T, Half& hw) {
  float A1[16], A2[8], A3[4];
  uint32_t w0 = 0u, w1 = 0u;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const float a0 = y[2 * i], b0 = y[2 * i + 1];
    A1[i] = fmaf(a0, a0, b0 * b0);
    const uint32_t k = sector16(a0, b0);
    if (i < 8)
      w0 |= k << (4 * i);
    else
      w1 |= k << (4 * (i - 8));
  }
  hw.l1[2 * cc] = w0;
  hw.l1[2 * cc + 1] = w1;
  uint32_t v2 = 0u;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    v2 |= code4(A1[2 * i], A1[2 * i + 1], T) << (2 * i);
    A2[i] = A1[2 * i] + A1[2 * i + 1];
  }
  hw.l2 |= v2 << (16 * cc);
  uint32_t v3 = 0u;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    v3 |= code4(A2[2 * i], A2[2 * i + 1], T + 3) << (2 * i);
    A3[i] = A2[2 * i] + A2[2 * i + 1];
  }
  hw.l3 |= v3 << (8 * cc);
  uint32_t v4 = 0u;
  float r4[2];
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    v4 |= code4(A3[2 * i], A3[2 * i + 1], T + 6) << (2 * i);
    r4[i] = sqrtf(A3[2 * i] + A3[2 * i + 1]);
  }
  hw.l4 |= v4 << (4 * cc);
  hw.r[cc] = (uint32_t)__half_as_ushort(__float2half_rn(r4[0])) |
             ((uint32_t)__half_as_ushort(__float2half_rn(r4[1])) << 16);
}

// y_hat of chunk cc of the half from its codes and 16-bit radii (the inverse transform);
// cs = (cos, sin) of the centroids: level 1 at [0, 16), level l >= 2 at 16 + 4 (l - 2)
__device__ __forceinline__ void rebuild_chunk(const Half& hw, int cc, uint32_t cs_s, float* yh) {
  auto cs = [&](int idx) {
    const uint2 v = lds_v2(cs_s + 8u * (uint32_t)idx);
    return make_float2(__uint_as_float(v.x), __uint_as_float(v.y));
  };
  const uint32_t rw = hw.r[cc];
  const float rh[2] = {__half2float(__ushort_as_half((unsigned short)(rw & 0xFFFFu))),
                       __half2float(__ushort_as_half((unsigned short)(rw >> 16)))};
  float q3[4], q2[8], q1[16];
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const float2 t = cs(24 + (int)((hw.l4 >> (4 * cc + 2 * i)) & 3u));
    q3[2 * i] = rh[i] * t.x;
    q3[2 * i + 1] = rh[i] * t.y;
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 t = cs(20 + (int)((hw.l3 >> (8 * cc + 2 * i)) & 3u));
    q2[2 * i] = q3[i] * t.x;
    q2[2 * i + 1] = q3[i] * t.y;
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float2 t = cs(16 + (int)((hw.l2 >> (16 * cc + 2 * i)) & 3u));
    q1[2 * i] = q2[i] * t.x;
    q1[2 * i + 1] = q2[i] * t.y;
  }
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const float2 t = cs((int)((hw.l1[2 * cc + (i >> 3)] >> (4 * (i & 7))) & 15u));
    yh[2 * i] = q1[i] * t.x;
    yh[2 * i + 1] = q1[i] * t.y;
  }
}

template <typename T, int MODE>
__global__ void __launch_bounds__(kThreads, 2)
    pq_kernel(const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_pi,
              const __grid_constant__ CUtensorMap map_o, PqArgs a) {
  using SM = Smem;
  constexpr bool kQ = MODE == PQ_QDQ;
  constexpr uint32_t kNcols = 256;
  constexpr uint32_t kIdPi = umma_idesc_f16(IsBf16<T>::value, IsBf16<T>::value, false, D, kRows);  // X Pi^T
  constexpr uint32_t kIdPiT = umma_idesc_f16(IsBf16<T>::value, IsBf16<T>::value, true, D, kRows);  // Y Pi

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* s_buf = smem + SM::buf_off;
  uint8_t* s_pi = smem + SM::pi_off;
  float2* s_cs = reinterpret_cast<float2*>(smem + SM::cs_off);
  float* s_tan = reinterpret_cast<float*>(smem + SM::tan_off);
  uint32_t* s_xchg = reinterpret_cast<uint32_t*>(smem + SM::xchg_off);
  uint64_t* bar_x = reinterpret_cast<uint64_t*>(smem + SM::bar_off);  // [2]
  uint64_t* bar_p = bar_x + 2;
  uint64_t* bar_m = bar_x + 3;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + SM::tmem_off);

  const int tid = threadIdx.x, warp = tid >> 5;
  const int r = tid & (kRows - 1);  // row in the tile = TMEM lane
  const int h = warp >> 2;          // half of the columns
  const int64_t n = a.n;
  const int64_t ntiles = (n + kRows - 1) / kRows;
  const uint32_t buf_s = smem_u32(s_buf), pi_s = smem_u32(s_pi), cs_s = smem_u32(s_cs);
  const int64_t ldc = a.ldc;
  // 16-byte code-word accesses when every row's words start 16-byte aligned
  const bool vec = (ldc & 3) == 0 &&
                   ((reinterpret_cast<uintptr_t>(kQ ? (const void*)a.codes_out : (const void*)a.codes_in) & 15u) == 0);

  if (tid == 0) {
    if (kQ) tma_prefetch_desc(&map_x);
    tma_prefetch_desc(&map_pi);
    tma_prefetch_desc(&map_o);
    mbar_init(bar_x, 1);
    mbar_init(bar_x + 1, 1);
    mbar_init(bar_p, 1);
    mbar_init(bar_m, 1);
    fence_barrier_init();
  }
  if (warp == 0) tmem_alloc(s_tmem, kNcols);
  // constants from the codebooks (boundaries: midpoints of neighbouring centroids)
  if (tid < kPqCentroids) {
    const float c = a.centroids[tid];
    s_cs[tid] = make_float2(cosf(c), sinf(c));
  } else if (tid >= 32 && tid < 32 + 9) {
    const int l = (tid - 32) / 3, j = (tid - 32) % 3;  // level l + 2, boundary j
    const float* c = a.centroids + 16 + 4 * l;
    const float t = tanf(0.5f * (c[j] + c[j + 1]));
    s_tan[3 * l + j] = t * t;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;
  const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
  const uint32_t tm_y = tmem + lane_off + 64u * (uint32_t)h, tm_x = tmem + 128u + lane_off + 64u * (uint32_t)h;

  if (tid == 0) {
    mbar_arrive_expect_tx(bar_p, kTileBytes);
    for (int b = 0; b < 2; ++b) tma_load_2d(s_pi + b * kBoxBytes, &map_pi, b * 64, 0, bar_p);
    if (kQ && (int64_t)blockIdx.x < ntiles) {
      mbar_arrive_expect_tx(bar_x, kTileBytes);
      for (int b = 0; b < 2; ++b)
        tma_load_2d(s_buf + b * kBoxBytes, &map_x, b * 64, (int32_t)((int64_t)blockIdx.x * kRows), bar_x);
    }
  }
  float Tq[9];
#pragma unroll
  for (int i = 0; i < 9; ++i) Tq[i] = s_tan[i];
  bool ok = __syncthreads_and(mbar_wait(bar_p, 0, a.status));
  uint32_t par_m = 0;

  auto mma = [&](uint32_t a_s, uint32_t tm_d, uint32_t idesc, bool mn_b) {  // thread 0
    tc_fence_after();
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const uint32_t akoff = (uint32_t)((kk >> 2) * kBoxBytes + (kk & 3) * 32);
      const uint32_t bkoff = mn_b ? (uint32_t)(kk * 16 * 128) : akoff;
      umma_f16(tm_d, umma_desc_sw128(a_s + akoff, 16, 1024),
               umma_desc_sw128(pi_s + bkoff, mn_b ? kBoxBytes : 16, 1024), idesc, kk > 0);
    }
    umma_commit(bar_m);
  };
  auto wait_mma = [&]() {
    const bool w = mbar_wait(bar_m, par_m, a.status);
    par_m ^= 1;
    tc_fence_after();
    return w;
  };

  // dequantize: the code words of this thread's half row of tile `t` (zeros past the last row), loaded
  // one tile ahead
  struct Raw {
    uint32_t l1[4], l2, w10, w11, r[2];
  };
  auto load_raw = [&](int64_t t, Raw& o) {
#pragma unroll
    for (int i = 0; i < 4; ++i) o.l1[i] = 0u;
    o.l2 = o.w10 = o.w11 = o.r[0] = o.r[1] = 0u;
    const int64_t row_ = t * kRows + r;
    if (t >= ntiles || row_ >= n) return;
    const uint32_t* src = a.codes_in + row_ * ldc;
    if (vec) {
      const uint4 l = __ldg(reinterpret_cast<const uint4*>(src + 4 * h));
      o.l1[0] = l.x, o.l1[1] = l.y, o.l1[2] = l.z, o.l1[3] = l.w;
      o.l2 = __ldg(src + 8 + h);
      const uint2 m = __ldg(reinterpret_cast<const uint2*>(src + 10));
      o.w10 = m.x, o.w11 = m.y;
      const uint2 q = __ldg(reinterpret_cast<const uint2*>(src + 12 + 2 * h));
      o.r[0] = q.x, o.r[1] = q.y;
    } else {
#pragma unroll
      for (int i = 0; i < 4; ++i) o.l1[i] = __ldg(src + 4 * h + i);
      o.l2 = __ldg(src + 8 + h);
      o.w10 = __ldg(src + 10), o.w11 = __ldg(src + 11);
      o.r[0] = __ldg(src + 12 + 2 * h), o.r[1] = __ldg(src + 13 + 2 * h);
    }
  };
  Raw raw_p;
  if constexpr (!kQ) load_raw(blockIdx.x, raw_p);

  int k = 0;
  for (int64_t tile = blockIdx.x; ok && tile < ntiles; tile += gridDim.x, ++k) {
    const int s = k & 1;
    uint8_t* tbuf = s_buf + s * kTileBytes;
    const uint32_t tbuf_s = buf_s + (uint32_t)(s * kTileBytes);
    const int64_t row0 = tile * kRows;
    const int rows = (int)(n - row0 < (int64_t)kRows ? n - row0 : (int64_t)kRows);
    const int64_t next = tile + gridDim.x;
    Half hw;
    hw.l2 = hw.l3 = hw.l4 = 0u;
    if constexpr (kQ) {
      if (tid == 0) {
        if (mbar_wait(bar_x + s, (uint32_t)(k >> 1) & 1u, a.status))
          mma(tbuf_s, tmem, kIdPi, false);  // y = Pi x per row
        else
          ok = false;
      }
      if (!wait_mma()) ok = false;
      if (tid == 0 && next < ntiles) {
        // the other buffer's x_hat store (previous tile) has been read: load the next tile's x into it
        bulk_wait_read<0>();
        mbar_arrive_expect_tx(bar_x + (s ^ 1), kTileBytes);
        for (int b = 0; b < 2; ++b)
          tma_load_2d(s_buf + (s ^ 1) * kTileBytes + b * kBoxBytes, &map_x, b * 64, (int32_t)(next * kRows),
                      bar_x + (s ^ 1));
      }
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        float y[32];
        tmem_ld32(tm_y + 32u * (uint32_t)cc, y);
        quantize_chunk(y, cc, Tq, hw);
      }
      if (h == 1) s_xchg[r] = hw.l3 | (hw.l4 << 16);
    } else {
      if (tid == 0) bulk_wait_read<1>();  // this buffer's store (two tiles back) has been read
      // this tile's words (loaded during the previous tile); the next tile's load starts now
      const Raw cur = raw_p;
      load_raw(next, raw_p);
#pragma unroll
      for (int i = 0; i < 4; ++i) hw.l1[i] = cur.l1[i];
      hw.l2 = cur.l2;
      hw.r[0] = cur.r[0], hw.r[1] = cur.r[1];
      hw.l3 = (cur.w10 >> (16 * h)) & 0xFFFFu;
      hw.l4 = (cur.w11 >> (8 * h)) & 0xFFu;
      __syncthreads();  // the buffer is free
    }
    // y_hat (the inverse transform of the codes and the 16-bit radii) as the second A operand
#pragma unroll
    for (int cc = 0; cc < 2; ++cc) {
      float yh[32];
      rebuild_chunk(hw, cc, cs_s, yh);
#pragma unroll
      for (int q = 0; q < 4; ++q)
        sts_v4(tbuf_s + sw128_chunk(r, 8 * h + 4 * cc + q, kBoxBytes), Elem<T>::pack(&yh[8 * q]));
    }
    fence_proxy_async_smem();
    tc_fence_before();
    ok = __syncthreads_and(ok);
    if (!ok) break;
    if (tid == 0) mma(tbuf_s, tmem + 128u, kIdPiT, true);  // x_hat = Pi^T y_hat per row
    if (kQ && a.codes_out && r < rows) {
      uint32_t* dst = a.codes_out + (row0 + r) * ldc;
      uint32_t w10 = 0u, w11 = 0u;
      if (h == 0) {
        const uint32_t x1 = s_xchg[r];
        w10 = hw.l3 | (x1 << 16);
        w11 = hw.l4 | (((x1 >> 16) & 0xFFu) << 8);
      }
      if (vec) {
        *reinterpret_cast<uint4*>(dst + 4 * h) = make_uint4(hw.l1[0], hw.l1[1], hw.l1[2], hw.l1[3]);
        dst[8 + h] = hw.l2;
        if (h == 0) *reinterpret_cast<uint2*>(dst + 10) = make_uint2(w10, w11);
        *reinterpret_cast<uint2*>(dst + 12 + 2 * h) = make_uint2(hw.r[0], hw.r[1]);
      } else {
#pragma unroll
        for (int i = 0; i < 4; ++i) dst[4 * h + i] = hw.l1[i];
        dst[8 + h] = hw.l2;
        if (h == 0) dst[10] = w10, dst[11] = w11;
        dst[12 + 2 * h] = hw.r[0], dst[13 + 2 * h] = hw.r[1];
      }
    }
    if (!wait_mma()) ok = false;
#pragma unroll
    for (int cc = 0; cc < 2; ++cc) {
      float v[32];
      tmem_ld32(tm_x + 32u * (uint32_t)cc, v);
#pragma unroll
      for (int q = 0; q < 4; ++q)
        sts_v4(tbuf_s + sw128_chunk(r, 8 * h + 4 * cc + q, kBoxBytes), Elem<T>::pack(&v[8 * q]));
    }
    fence_proxy_async_smem();
    tc_fence_before();
    ok = __syncthreads_and(ok);
    if (!ok) break;
    if (tid == 0) {
      for (int b = 0; b < 2; ++b) tma_store_2d(&map_o, b * 64, (int32_t)row0, tbuf + b * kBoxBytes);
      bulk_commit();
    }
  }
  // the stores have read their shared-memory sources; their writes complete with the grid
  if (tid == 0) bulk_wait_read<0>();
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
  kern<<<(unsigned)grid, kThreads, Smem::alloc, st>>>(mx, mp, mo, a);
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
