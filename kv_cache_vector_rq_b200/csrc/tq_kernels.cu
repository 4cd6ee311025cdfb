// TurboQuant kernels for sm_100a: dense rotation and QJL projection on the
// 5th-generation tensor cores (tcgen05.mma, accumulators in TMEM).
//
// Method (arXiv 2504.19874 summary page, "方法", Algorithms 1 and 2;
// "TurboQuant 论文解读", "随机旋转（Lemma 1）" and "QJL 内积无偏估计（Theorem 2）";
// "TurboQuant + RotorQuant", "How TurboQuant Works"):
//   u = x / ||x||, y = Pi u, code_i = nearest Lloyd-Max centroid of y_i,
//   x_hat = ||x|| Pi^T c_hat                                          (mse)
//   (b-1)-bit mse codes, r = y - c_hat (rotated residual), gamma = ||r||,
//   s = sign(T r) with S = T Pi, x_hat = ||x|| Pi^T (c_hat + sqrt(pi/2)/m gamma T^T s)   (prod)
//
// B200 design. Pi (and T) stay resident in shared memory as 128-byte-swizzled tiles
// that serve as the MMA B operand both K-major (y = Pi u, T r) and MN-major (Pi^T c,
// T^T s). The x tile arrives by TMA in the same swizzled layout and is the A operand
// directly. One thread issues tcgen05.mma (M = 128, N = d, K = 16 steps) into TMEM;
// the threads then read their rows (one TMEM lane per row) with tcgen05.ld, quantize
// on the FMA pipe, and write the next A operand (centroids, or the residual for the
// sketch) back into the tile buffer, which finally holds x_hat for the TMA store.
//  * tq_mse_kernel (the mse modes): 256 threads, two per row (64 columns each), two
//    tile buffers so the next tile's load lands while this tile is quantized.
//  * tq_prod_kernel (prod quantize): 256 threads, two per row; Pi and T leave room for
//    one tile buffer at two CTAs per SM, so the sketch operand goes to tensor memory
//    and the buffer takes the next tile's x as soon as the first product has read it.
//  * tq_dq_prod_kernel (prod dequantize): 256 threads, two per row; the sign operand in tensor
//    memory, the corrected centroids in the tile buffer, one tile at a time.
// Two CTAs share an SM (256 TMEM columns each), so one CTA's MMAs overlap the other's
// epilogue.

#include <cuda_runtime.h>

#include <cstdlib>
#include <type_traits>

#include "bisect.cuh"
#include "kvrq_device.cuh"
#include "tq_launch.h"

namespace kvrq {
namespace tq {

constexpr int kRows = 128;
constexpr int D = 128;                            // head dimension handled by this kernel (= m)
constexpr int kBoxBytes = kRows * 128;            // one 64-column box of 128 rows
constexpr int kTileBytes = 2 * kBoxBytes;         // 128 x 128 16-bit elements
constexpr float kShift = 9.313225746154785e-10f;  // 2^-30
constexpr float kWindow0 = 8388608.0f;            // 2^23
constexpr float kSketchScale = 256.0f;            // residual scale before rounding to fp16

template <int BITS>
struct Codes {
  static constexpr int K = 1 << BITS;
  static constexpr int H = K / 2;
  static constexpr int NC = D;
  static constexpr int W = (NC * BITS + 31) / 32;
  static constexpr int CPW = 23 / BITS;
  static constexpr int NWIN = (NC + CPW - 1) / CPW;
};


// Positive-side quantizer constants (see rq_kernels.cu for the construction):
// sc[j] = -tau_{j+1} * B, chain of unit centroids c[H] + sum step_j * dl[j].
template <int BITS>
__device__ __forceinline__ void build_consts(const float* __restrict__ centroids, float* sc, float* mag, float* cf,
                                             float* bscale) {
  constexpr int K = 1 << BITS, H = K / 2;
  const int t = threadIdx.x;
  // B = 2^(48 - floor(log2 tau_min)) keeps every step exactly 0 or 1
  float tau_min = 1.f;
  if (H > 1) tau_min = 0.5f * (centroids[H] + centroids[H + 1]);
  const int e = (int)((__float_as_uint(tau_min) >> 23) & 0xFF) - 127;
  const float B = __uint_as_float((uint32_t)(127 + 48 - e) << 23);  // exactly 2^(48 - e)
  if (t == 0) *bscale = B;
  if (t < H) mag[t] = centroids[H + t];
  if (t < H - 1) sc[t] = -(0.5f * (centroids[H + t] + centroids[H + 1 + t])) * B;
  // centroid table as the quantizer builds it: c[H + j] = c[H] + (c[H+1] - c[H]) + ... (rounded
  // step by step), c[H - 1 - j] = -c[H + j]; so quantize-then-dequantize equals the fused path
  if (t == 0) {
    float ch = centroids[H];
    for (int j = 0; j < H; ++j) {
      if (j > 0) ch = __fadd_rn(ch, __fsub_rn(centroids[H + j], centroids[H + j - 1]));
      cf[H + j] = ch;
      cf[H - 1 - j] = -ch;
    }
  }
}

template <typename T>
struct IsBf16 {
  static constexpr bool value = std::is_same<T, __nv_bfloat16>::value;
};

// ============================================================================ mse, two threads per row
// TurboQuant-mse at d = 128 (quantize, roundtrip, dequantize) with 256-thread CTAs: thread (row r,
// half h = warp / 4) owns columns 64h .. 64h + 63 of its row (TMEM lane r), so a warp's chain is
// half as long and an SM holds twice the warps. The row norm is the sum of the two halves' sums of
// squares, exchanged through shared memory under a barrier of the two warps that share the rows.
// Two tile buffers alternate: the next tile's x is loaded as soon as this tile's first product has
// read its own, and lands while this tile is quantized; the centroid operand of the second product
// is written over x, and x_hat over the centroids. A half row holds 64 codes, whole code words.
constexpr int kThreadsM = 256;

template <int BITS>
struct HalfRow {
  static constexpr int CPW = 23 / BITS;                 // codes per mantissa window
  static constexpr int NWH = (64 + CPW - 1) / CPW;      // windows of a half row
  static constexpr int WH = 2 * BITS;                   // code words of a half row
};

struct SmemM {
  static constexpr int buf_off = 0;                         // two tiles
  static constexpr int pi_off = 2 * kTileBytes;
  static constexpr int cb_off = pi_off + kTileBytes;        // 64 floats: sc, mag, cf, bscale
  static constexpr int part_off = cb_off + 64 * 4;          // float [2][kRows]: the halves' sums of squares
  static constexpr int bar_off = part_off + 2 * kRows * 4;  // x[2], params, mma
  static constexpr int tmem_off = bar_off + 4 * 8;
  static constexpr int bytes = tmem_off + 16;
  static constexpr int alloc = bytes + 1024;
};
static_assert(2 * (SmemM::alloc + 1024) <= 228 * 1024, "two CTAs per SM");

// barrier of the two warps (w, w + 4) whose threads share the rows 32 (w & 3) ..
__device__ __forceinline__ void pair_sync(int warp) {
  asm volatile("bar.sync %0, %1;" ::"r"(1 + (warp & 3)), "r"(64) : "memory");
}

template <typename T, int BITS, int MODE>
__global__ void __launch_bounds__(kThreadsM, 2)
    tq_mse_kernel(const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_pi,
                  const __grid_constant__ CUtensorMap map_o, TqArgs a) {
  using HR = HalfRow<BITS>;
  using SM = SmemM;
  constexpr int H = Codes<BITS>::H, CPW = HR::CPW, NWH = HR::NWH, WH = HR::WH;
  constexpr bool kQ = MODE != TQ_DQ_MSE;
  constexpr bool kOut = MODE != TQ_MSE_Q;
  constexpr uint32_t kNcols = 256;
  constexpr uint32_t kIdPi = umma_idesc_f16(IsBf16<T>::value, IsBf16<T>::value, false, D, kRows);  // X Pi^T
  constexpr uint32_t kIdPiT = umma_idesc_f16(IsBf16<T>::value, IsBf16<T>::value, true, D, kRows);  // C Pi

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* s_buf = smem + SM::buf_off;
  uint8_t* s_pi = smem + SM::pi_off;
  float* s_sc = reinterpret_cast<float*>(smem + SM::cb_off);
  float* s_mag = s_sc + 16;
  float* s_cf = s_sc + 32;
  float* s_bscale = s_sc + 48;
  float* s_part = reinterpret_cast<float*>(smem + SM::part_off);
  uint64_t* bar_x = reinterpret_cast<uint64_t*>(smem + SM::bar_off);  // [2]
  uint64_t* bar_p = bar_x + 2;
  uint64_t* bar_m = bar_x + 3;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + SM::tmem_off);

  const int tid = threadIdx.x, warp = tid >> 5;
  const int r = tid & (kRows - 1);  // row in the tile = TMEM lane
  const int h = warp >> 2;          // half of the columns
  const int64_t n = a.n;
  const int64_t ntiles = (n + kRows - 1) / kRows;
  const uint32_t buf_s = smem_u32(s_buf), pi_s = smem_u32(s_pi);
  // 8-byte code-word accesses when every half row's words start 8-byte aligned
  const bool vec = (a.ldc & 1) == 0 &&
                   ((reinterpret_cast<uintptr_t>(kQ ? (const void*)a.codes_out : (const void*)a.codes_in) & 7u) == 0);

  // launched with programmatic stream serialization: every global access follows this wait
  grid_dep_wait();
  grid_dep_launch();
  if (tid == 0) {
    if (kQ) tma_prefetch_desc(&map_x);
    tma_prefetch_desc(&map_pi);
    if (kOut) tma_prefetch_desc(&map_o);
    mbar_init(bar_x, 1);
    mbar_init(bar_x + 1, 1);
    mbar_init(bar_p, 1);
    mbar_init(bar_m, 1);
    fence_barrier_init();
  }
  if (warp == 0) tmem_alloc(s_tmem, kNcols);
  build_consts<BITS>(a.centroids, s_sc, s_mag, s_cf, s_bscale);
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
  const float Bs = *s_bscale;
  float dl[H > 1 ? H - 1 : 1], sc[H > 1 ? H - 1 : 1];
#pragma unroll
  for (int j = 0; j < H - 1; ++j) {
    dl[j] = __fsub_rn(s_mag[j + 1], s_mag[j]);
    sc[j] = s_sc[j];
  }
  const float mn0 = s_mag[0];
  // b >= 3: binary search over the boundaries (one saturating step per code bit); the centroid table
  // of the dequantize side is rebuilt from the same magnitude sequence, so both sides give the same bits
  constexpr bool kBisect = BITS >= 3;
  Bisect<kBisect ? BITS : 3> bs;
  if constexpr (kBisect) {
    bs.thresholds(sc);
    bs.magnitudes(s_mag);
  }
  bool ok = mbar_wait(bar_p, 0, a.status);
  if constexpr (kBisect) {
    if (tid < H) {
      const float m = bs.mag(tid);
      s_cf[H + tid] = m;
      s_cf[H - 1 - tid] = -m;
    }
  }
  ok = __syncthreads_and(ok);
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

  // dequantize: this thread's half row of tile `t` (zeros past the last row), loaded one tile ahead
  auto load_codes = [&](int64_t t, uint32_t (&wc_)[WH], float& nrm_) {
#pragma unroll
    for (int w = 0; w < WH; ++w) wc_[w] = 0u;
    nrm_ = 0.f;
    const int64_t row_ = t * kRows + r;
    if (t >= ntiles || row_ >= n) return;
    const uint32_t* src = a.codes_in + row_ * a.ldc + WH * h;
    if (vec) {
#pragma unroll
      for (int w = 0; w < WH; w += 2) {
        const uint2 v = __ldg(reinterpret_cast<const uint2*>(src + w));
        wc_[w] = v.x, wc_[w + 1] = v.y;
      }
    } else {
#pragma unroll
      for (int w = 0; w < WH; ++w) wc_[w] = __ldg(src + w);
    }
    nrm_ = __ldg(a.norms_in + row_ * a.ldn);
  };
  uint32_t wc_p[WH];
  float nrm_p = 0.f;
  if constexpr (!kQ) load_codes(blockIdx.x, wc_p, nrm_p);

  int k = 0;
  for (int64_t tile = blockIdx.x; ok && tile < ntiles; tile += gridDim.x, ++k) {
    const int s = k & 1;
    uint8_t* tbuf = s_buf + s * kTileBytes;
    const uint32_t tbuf_s = buf_s + (uint32_t)(s * kTileBytes);
    const int64_t row0 = tile * kRows;
    const int rows = (int)(n - row0 < (int64_t)kRows ? n - row0 : (int64_t)kRows);
    const int64_t next = tile + gridDim.x;
    const bool live = r < rows;
    const int64_t row = row0 + r;
    float nrm = 0.f;
    uint32_t wc[WH];
#pragma unroll
    for (int w = 0; w < WH; ++w) wc[w] = 0u;
    auto put = [&](int j, const float* v) {
      sts_v4(tbuf_s + sw128_chunk(r, j, kBoxBytes), Elem<T>::pack(v));
    };
    auto store_outputs = [&]() {  // code words and norm of this half row
      if (!kQ || !live) return;
      const int64_t orow = a.out_rows ? a.out_rows[row] : row;
      if (a.codes_out) {
        uint32_t* dst = a.codes_out + orow * a.ldc + WH * h;
        if (vec) {
#pragma unroll
          for (int w = 0; w < WH; w += 2) *reinterpret_cast<uint2*>(dst + w) = make_uint2(wc[w], wc[w + 1]);
        } else {
#pragma unroll
          for (int w = 0; w < WH; ++w) dst[w] = wc[w];
        }
      }
      if (h == 0 && a.norms_out) a.norms_out[orow * a.ldn] = nrm;
    };

    if constexpr (kQ) {
      // every thread reads x from the tile (its half's sum of squares), so every thread waits for it
      const bool landed = mbar_wait(bar_x + s, (uint32_t)(k >> 1) & 1u, a.status);
      if (!landed) ok = false;
      if (tid == 0 && landed) mma(tbuf_s, tmem, kIdPi, false);  // y = Pi x per row
      // this half's sum of squares from the tile while the MMA runs
      float2 acc[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) acc[q] = make_float2(0.f, 0.f);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if constexpr (std::is_same<T, __half>::value) {  // fp16 squares straight into the fp32 sums
          const uint4 c = lds_v4(tbuf_s + sw128_chunk(r, 8 * h + j, kBoxBytes));
          const uint32_t cw[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
          for (int q = 0; q < 4; ++q) sq_acc_f16x2(cw[q], acc[q].x, acc[q].y);
        } else {
          float f[8];
          Elem<T>::unpack(lds_v4(tbuf_s + sw128_chunk(r, 8 * h + j, kBoxBytes)), f);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float2 v = make_float2(f[2 * q], f[2 * q + 1]);
            acc[q] = __ffma2_rn(v, v, acc[q]);
          }
        }
      }
      s_part[h * kRows + r] =
          ((acc[0].x + acc[1].x) + (acc[2].x + acc[3].x)) + ((acc[0].y + acc[1].y) + (acc[2].y + acc[3].y));
      if (!wait_mma()) ok = false;
      pair_sync(warp);
      nrm = sqrtf(s_part[r] + s_part[kRows + r]);
      if (tid == 0 && next < ntiles) {
        // the other buffer's x_hat store (previous tile) has been read: load the next tile's x into it
        bulk_wait_read<0>();
        mbar_arrive_expect_tx(bar_x + (s ^ 1), kTileBytes);
        for (int b = 0; b < 2; ++b)
          tma_load_2d(s_buf + (s ^ 1) * kTileBytes + b * kBoxBytes, &map_x, b * 64, (int32_t)(next * kRows),
                      bar_x + (s ^ 1));
      }
      const float srow = nrm > 0.f ? __fdiv_rn(Bs, nrm) : 0.f;
      const float shift = -fmaf(kShift, nrm, 0x1p-126f);
      float win[NWH];
#pragma unroll
      for (int w = 0; w < NWH; ++w) win[w] = kWindow0;
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        float y[32];
        tmem_ld32(tm_y + 32u * (uint32_t)cc, y);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
        float w_out[8];
#pragma unroll
        for (int i = 8 * q; i < 8 * q + 8; i += 2) {
          const float2 Y = make_float2(y[i] + shift, y[i + 1] + shift);
          float2 m2 = make_float2(mn0, mn0), cnt = make_float2(0.5f, 0.5f);
          if constexpr (kBisect) {
            bs(make_float2(fabsf(Y.x), fabsf(Y.y)), srow, m2, cnt);
          } else {
#pragma unroll
            for (int j = 0; j < H - 1; ++j) {
              const float2 st = make_float2(fma_sat(fabsf(Y.x), srow, sc[j]), fma_sat(fabsf(Y.y), srow, sc[j]));
              m2 = __ffma2_rn(st, make_float2(dl[j], dl[j]), m2);
              cnt = __fadd2_rn(cnt, st);
            }
          }
          const float2 sg = make_float2(sign_one(Y.x), sign_one(Y.y));
          const float2 code = __ffma2_rn(sg, cnt, make_float2(H - 0.5f, H - 0.5f));
          const int k0 = 32 * cc + i, k1 = k0 + 1;  // code index in the half row
          win[k0 / CPW] = fmaf(code.x, (float)(1u << (BITS * (k0 % CPW))), win[k0 / CPW]);
          win[k1 / CPW] = fmaf(code.y, (float)(1u << (BITS * (k1 % CPW))), win[k1 / CPW]);
          if constexpr (kOut) {
            const float2 chat = __fmul2_rn(m2, sg);  // unit-scale centroid
            w_out[i - 8 * q] = chat.x;
            w_out[i + 1 - 8 * q] = chat.y;
          }
        }
        if constexpr (kOut) put(8 * h + 4 * cc + q, w_out);
        }
      }
#pragma unroll
      for (int w = 0; w < NWH; ++w) {
        const uint32_t v = __float_as_uint(win[w]) & 0x7fffffu;
        const int bo = w * CPW * BITS;
        wc[bo >> 5] |= v << (bo & 31);
        if ((bo & 31) + CPW * BITS > 32 && (bo >> 5) + 1 < WH) wc[(bo >> 5) + 1] |= v >> (32 - (bo & 31));
      }
    } else {
      if (tid == 0) bulk_wait_read<1>();  // this buffer's store (two tiles back) has been read
      // this tile's codes and norm (loaded during the previous tile); the next tile's load starts now
#pragma unroll
      for (int w = 0; w < WH; ++w) wc[w] = wc_p[w];
      nrm = nrm_p;
      load_codes(next, wc_p, nrm_p);
      auto code_at = [&](int kl) -> uint32_t {
        const int bit = kl * BITS, word = bit >> 5, sh = bit & 31;
        uint32_t v = wc[word] >> sh;
        if (sh + BITS > 32) v |= wc[word + 1] << (32 - sh);
        return v & ((1u << BITS) - 1u);
      };
      __syncthreads();  // the buffer is free
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        float v[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = s_cf[code_at(32 * cc + i)];
#pragma unroll
        for (int q = 0; q < 4; ++q) put(8 * h + 4 * cc + q, &v[8 * q]);
      }
    }

    if constexpr (kOut) {
      fence_proxy_async_smem();
      tc_fence_before();
      ok = __syncthreads_and(ok);
      if (!ok) break;
      if (tid == 0) mma(tbuf_s, tmem + 128u, kIdPiT, true);  // Pi^T c_hat per row
      store_outputs();
      if (!wait_mma()) ok = false;
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        float v[32];
        tmem_ld32(tm_x + 32u * (uint32_t)cc, v);
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] *= nrm;
#pragma unroll
        for (int q = 0; q < 4; ++q) put(8 * h + 4 * cc + q, &v[8 * q]);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      ok = __syncthreads_and(ok);
      if (!ok) break;
      if (tid == 0) {
        for (int b = 0; b < 2; ++b) tma_store_2d(&map_o, b * 64, (int32_t)row0, tbuf + b * kBoxBytes);
        bulk_commit();
      }
    } else {
      store_outputs();
      tc_fence_before();  // this tile's TMEM reads precede the next tile's product
      ok = __syncthreads_and(ok);
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

// ============================================================================ prod, two threads per row
// TurboQuant-prod quantize at d = 128 with 256-thread CTAs, two threads per row as in tq_mse_kernel.
// Pi and T stay resident (64 KB), which leaves one tile buffer at two CTAs per SM; the sketch's A
// operand, fp16(2^8 r), goes to tensor memory (64 columns beside the 128 of y), so the x buffer is
// free as soon as the first product and the norm pass have read it, and the next tile's load is
// issued then: it lands while this tile is quantized, sketched and stored. T r reuses y's columns.
struct SmemP {
  static constexpr int buf_off = 0;                          // one tile
  static constexpr int pi_off = kTileBytes;
  static constexpr int t_off = 2 * kTileBytes;
  static constexpr int cb_off = 3 * kTileBytes;              // 64 floats: sc, mag, cf, bscale
  static constexpr int part_off = cb_off + 64 * 4;           // float [2][kRows]: halves' sums of squares
  static constexpr int gpart_off = part_off + 2 * kRows * 4;  // float [2][kRows]: halves' ||r||^2
  static constexpr int bar_off = gpart_off + 2 * kRows * 4;  // x, params, mma
  static constexpr int tmem_off = bar_off + 3 * 8;
  static constexpr int bytes = tmem_off + 16;
  static constexpr int alloc = bytes + 1024;
};
static_assert(2 * (SmemP::alloc + 1024) <= 228 * 1024, "two CTAs per SM");

template <typename T, int BITS>
__global__ void __launch_bounds__(kThreadsM, 2)
    tq_prod_kernel(const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_pi,
                   const __grid_constant__ CUtensorMap map_t, TqArgs a) {
  using HR = HalfRow<BITS>;
  using SM = SmemP;
  constexpr int H = Codes<BITS>::H, CPW = HR::CPW, NWH = HR::NWH, WH = HR::WH;
  constexpr uint32_t kNcols = 256;  // y (then T r): 0 .. 127; the sketch operand: 128 .. 191
  constexpr uint32_t kIdPi = umma_idesc_f16(IsBf16<T>::value, IsBf16<T>::value, false, D, kRows);  // X Pi^T
  constexpr uint32_t kIdT = umma_idesc_f16(false, false, false, D, kRows);                          // rho T^T

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* s_buf = smem + SM::buf_off;
  uint8_t* s_pi = smem + SM::pi_off;
  uint8_t* s_t = smem + SM::t_off;
  float* s_sc = reinterpret_cast<float*>(smem + SM::cb_off);
  float* s_mag = s_sc + 16;
  float* s_cf = s_sc + 32;
  float* s_bscale = s_sc + 48;
  float* s_part = reinterpret_cast<float*>(smem + SM::part_off);
  float* s_gpart = reinterpret_cast<float*>(smem + SM::gpart_off);
  uint64_t* bar_x = reinterpret_cast<uint64_t*>(smem + SM::bar_off);
  uint64_t* bar_p = bar_x + 1;
  uint64_t* bar_m = bar_x + 2;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + SM::tmem_off);

  const int tid = threadIdx.x, warp = tid >> 5;
  const int r = tid & (kRows - 1);  // row in the tile = TMEM lane
  const int h = warp >> 2;          // half of the columns
  const int64_t n = a.n;
  const int64_t ntiles = (n + kRows - 1) / kRows;
  const uint32_t buf_s = smem_u32(s_buf), pi_s = smem_u32(s_pi), t_s = smem_u32(s_t);
  constexpr int NS = D / 32;  // sign words per row
  const bool vec = (a.ldc & 1) == 0 && (reinterpret_cast<uintptr_t>(a.codes_out) & 7u) == 0;
  const bool svec = (a.lds & 1) == 0 && (reinterpret_cast<uintptr_t>(a.signs_out) & 7u) == 0;

  // launched with programmatic stream serialization: every global access follows this wait
  grid_dep_wait();
  grid_dep_launch();
  if (tid == 0) {
    tma_prefetch_desc(&map_x);
    tma_prefetch_desc(&map_pi);
    tma_prefetch_desc(&map_t);
    mbar_init(bar_x, 1);
    mbar_init(bar_p, 1);
    mbar_init(bar_m, 1);
    fence_barrier_init();
  }
  if (warp == 0) tmem_alloc(s_tmem, kNcols);
  build_consts<BITS>(a.centroids, s_sc, s_mag, s_cf, s_bscale);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;
  const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
  const uint32_t tm_y = tmem + lane_off + 64u * (uint32_t)h;                // this half's y (then T r) columns
  const uint32_t tm_rho = tmem + 128u + lane_off + 32u * (uint32_t)h;       // this half's sketch operand words

  if (tid == 0) {
    mbar_arrive_expect_tx(bar_p, 2 * kTileBytes);
    for (int b = 0; b < 2; ++b) tma_load_2d(s_pi + b * kBoxBytes, &map_pi, b * 64, 0, bar_p);
    for (int b = 0; b < 2; ++b) tma_load_2d(s_t + b * kBoxBytes, &map_t, b * 64, 0, bar_p);
    if ((int64_t)blockIdx.x < ntiles) {
      mbar_arrive_expect_tx(bar_x, kTileBytes);
      for (int b = 0; b < 2; ++b)
        tma_load_2d(s_buf + b * kBoxBytes, &map_x, b * 64, (int32_t)((int64_t)blockIdx.x * kRows), bar_x);
    }
  }
  const float Bs = *s_bscale;
  float dl[H > 1 ? H - 1 : 1], sc[H > 1 ? H - 1 : 1];
#pragma unroll
  for (int j = 0; j < H - 1; ++j) {
    dl[j] = __fsub_rn(s_mag[j + 1], s_mag[j]);
    sc[j] = s_sc[j];
  }
  const float mn0 = s_mag[0];
  constexpr bool kBisect = BITS >= 3;
  Bisect<kBisect ? BITS : 3> bs;
  if constexpr (kBisect) {
    bs.thresholds(sc);
    bs.magnitudes(s_mag);
  }
  bool ok = __syncthreads_and(mbar_wait(bar_p, 0, a.status));
  uint32_t par_m = 0;

  auto wait_mma = [&]() {
    const bool w = mbar_wait(bar_m, par_m, a.status);
    par_m ^= 1;
    tc_fence_after();
    return w;
  };

  int k = 0;
  for (int64_t tile = blockIdx.x; ok && tile < ntiles; tile += gridDim.x, ++k) {
    const int64_t row0 = tile * kRows;
    const int rows = (int)(n - row0 < (int64_t)kRows ? n - row0 : (int64_t)kRows);
    const int64_t next = tile + gridDim.x;
    const bool live = r < rows;
    const int64_t row = row0 + r;

    // every thread reads x from the tile (its half's sum of squares), so every thread waits for it
    const bool landed = mbar_wait(bar_x, (uint32_t)k & 1u, a.status);
    if (!landed) ok = false;
    if (tid == 0 && landed) {  // y = Pi x per row
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t koff = (uint32_t)((kk >> 2) * kBoxBytes + (kk & 3) * 32);
        umma_f16(tmem, umma_desc_sw128(buf_s + koff, 16, 1024), umma_desc_sw128(pi_s + koff, 16, 1024), kIdPi,
                 kk > 0);
      }
      umma_commit(bar_m);
    }
    float2 acc[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) acc[q] = make_float2(0.f, 0.f);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if constexpr (std::is_same<T, __half>::value) {  // fp16 squares straight into the fp32 sums
        const uint4 c = lds_v4(buf_s + sw128_chunk(r, 8 * h + j, kBoxBytes));
        const uint32_t cw[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) sq_acc_f16x2(cw[q], acc[q].x, acc[q].y);
      } else {
        float f[8];
        Elem<T>::unpack(lds_v4(buf_s + sw128_chunk(r, 8 * h + j, kBoxBytes)), f);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float2 v = make_float2(f[2 * q], f[2 * q + 1]);
          acc[q] = __ffma2_rn(v, v, acc[q]);
        }
      }
    }
    s_part[h * kRows + r] =
        ((acc[0].x + acc[1].x) + (acc[2].x + acc[3].x)) + ((acc[0].y + acc[1].y) + (acc[2].y + acc[3].y));
    if (!wait_mma()) ok = false;
    __syncthreads();  // every half's sum is in, and no thread reads x any more
    const float nrm = sqrtf(s_part[r] + s_part[kRows + r]);
    if (tid == 0 && next < ntiles) {  // the product and the norm pass have read the buffer
      mbar_arrive_expect_tx(bar_x, kTileBytes);
      for (int b = 0; b < 2; ++b)
        tma_load_2d(s_buf + b * kBoxBytes, &map_x, b * 64, (int32_t)(next * kRows), bar_x);
    }

    const float srow = nrm > 0.f ? __fdiv_rn(Bs, nrm) : 0.f;
    const float shift = -fmaf(kShift, nrm, 0x1p-126f);
    const float rn = nrm > 0.f ? __frcp_rn(nrm) : 0.f;
    float win[NWH];
#pragma unroll
    for (int w = 0; w < NWH; ++w) win[w] = kWindow0;
    float gs = 0.f;
#pragma unroll
    for (int cc = 0; cc < 4; ++cc) {  // 16 columns at a time
      float y[16];
      tmem_ld16(tm_y + 16u * (uint32_t)cc, y);
      uint32_t rho[8];  // fp16(2^8 r) pairs of these columns
#pragma unroll
      for (int i = 0; i < 16; i += 2) {
        const float2 Y = make_float2(y[i] + shift, y[i + 1] + shift);
        float2 m2 = make_float2(mn0, mn0), cnt = make_float2(0.5f, 0.5f);
        if constexpr (kBisect) {
          bs(make_float2(fabsf(Y.x), fabsf(Y.y)), srow, m2, cnt);
        } else {
#pragma unroll
          for (int j = 0; j < H - 1; ++j) {
            const float2 st = make_float2(fma_sat(fabsf(Y.x), srow, sc[j]), fma_sat(fabsf(Y.y), srow, sc[j]));
            m2 = __ffma2_rn(st, make_float2(dl[j], dl[j]), m2);
            cnt = __fadd2_rn(cnt, st);
          }
        }
        const float2 sg = make_float2(sign_one(Y.x), sign_one(Y.y));
        const float2 chat = __fmul2_rn(m2, sg);  // unit-scale centroid
        const float2 code = __ffma2_rn(sg, cnt, make_float2(H - 0.5f, H - 0.5f));
        const int k0 = 16 * cc + i, k1 = k0 + 1;  // code index in the half row
        win[k0 / CPW] = fmaf(code.x, (float)(1u << (BITS * (k0 % CPW))), win[k0 / CPW]);
        win[k1 / CPW] = fmaf(code.y, (float)(1u << (BITS * (k1 % CPW))), win[k1 / CPW]);
        // rotated unit residual r = y / ||x|| - c_hat
        const float2 rr = __ffma2_rn(make_float2(y[i], y[i + 1]), make_float2(rn, rn), make_float2(-chat.x, -chat.y));
        gs = fmaf(rr.x, rr.x, fmaf(rr.y, rr.y, gs));
        const __half2 hp = __floats2half2_rn(rr.x * kSketchScale, rr.y * kSketchScale);
        rho[i / 2] = *reinterpret_cast<const uint32_t*>(&hp);
      }
      tmem_st8(tm_rho + 8u * (uint32_t)cc, rho);
    }
    s_gpart[h * kRows + r] = gs;
    uint32_t wc[WH];
#pragma unroll
    for (int w = 0; w < WH; ++w) wc[w] = 0u;
#pragma unroll
    for (int w = 0; w < NWH; ++w) {
      const uint32_t v = __float_as_uint(win[w]) & 0x7fffffu;
      const int bo = w * CPW * BITS;
      wc[bo >> 5] |= v << (bo & 31);
      if ((bo & 31) + CPW * BITS > 32 && (bo >> 5) + 1 < WH) wc[(bo >> 5) + 1] |= v >> (32 - (bo & 31));
    }
    tmem_wait_st();
    tc_fence_before();
    ok = __syncthreads_and(ok);  // the operand is complete and y has been read
    if (!ok) break;
    if (tid == 0) {  // T r per row, into y's columns
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t koff = (uint32_t)((kk >> 2) * kBoxBytes + (kk & 3) * 32);
        umma_f16_ts(tmem, tmem + 128u + (uint32_t)(8 * kk), umma_desc_sw128(t_s + koff, 16, 1024), kIdT, kk > 0);
      }
      umma_commit(bar_m);
    }
    const int64_t orow = live ? (a.out_rows ? a.out_rows[row] : row) : 0;
    if (live) {
      if (a.codes_out) {
        uint32_t* dst = a.codes_out + orow * a.ldc + WH * h;
        if (vec) {
#pragma unroll
          for (int w = 0; w < WH; w += 2) *reinterpret_cast<uint2*>(dst + w) = make_uint2(wc[w], wc[w + 1]);
        } else {
#pragma unroll
          for (int w = 0; w < WH; ++w) dst[w] = wc[w];
        }
      }
      if (h == 0) {
        if (a.norms_out) a.norms_out[orow * a.ldn] = nrm;
        if (a.gammas_out) a.gammas_out[orow * a.ldn] = sqrtf(s_gpart[r] + s_gpart[kRows + r]);
      }
    }
    if (!wait_mma()) ok = false;
    uint32_t sw[2];
#pragma unroll
    for (int cc = 0; cc < 2; ++cc) {
      float z[32];
      tmem_ld32(tm_y + 32u * (uint32_t)cc, z);
      uint32_t bits = 0;
#pragma unroll
      for (int i = 0; i < 32; ++i) bits |= (z[i] >= 0.f ? 1u : 0u) << i;  // sign(0) = +1
      sw[cc] = bits;
    }
    if (live && a.signs_out) {
      uint32_t* dst = a.signs_out + orow * a.lds + (NS / 2) * h;
      if (svec) *reinterpret_cast<uint2*>(dst) = make_uint2(sw[0], sw[1]);
      else dst[0] = sw[0], dst[1] = sw[1];
    }
    tc_fence_before();
    ok = __syncthreads_and(ok);  // T r has been read before the next tile's product overwrites it
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kNcols);
  }
}

// ============================================================================ prod dequantize, two threads per row
// x_hat = ||x|| Pi^T (c_hat + sqrt(pi/2)/m gamma T^T s) at d = 128 with 256-thread CTAs, two threads per
// row. Per tile each thread writes its half of the +-1 sign operand (fp16 pairs) into tensor memory,
// the A of T^T s (MN-major T); reads T^T s back, adds its centroids (the quantizer's magnitude
// sequence), and writes the corrected centroids w into the tile buffer, the A of Pi^T w; x_hat goes
// back over w and leaves by TMA. Pi and T resident (64 KB) and one tile buffer: two CTAs per SM.
template <typename T, int BITS>
__global__ void __launch_bounds__(kThreadsM, 2)
    tq_dq_prod_kernel(const __grid_constant__ CUtensorMap map_pi, const __grid_constant__ CUtensorMap map_t,
                      const __grid_constant__ CUtensorMap map_o, TqArgs a) {
  using HR = HalfRow<BITS>;
  using SM = SmemP;
  constexpr int H = Codes<BITS>::H, WH = HR::WH;
  constexpr int NS = D / 32;  // sign words per row
  constexpr uint32_t kNcols = 256;  // T^T s, then Pi^T w: 0 .. 127; the sign operand: 128 .. 191
  constexpr uint32_t kIdPiT = umma_idesc_f16(IsBf16<T>::value, IsBf16<T>::value, true, D, kRows);  // W Pi
  constexpr uint32_t kIdTT = umma_idesc_f16(false, false, true, D, kRows);                          // S T

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* s_pi = smem + SM::pi_off;
  uint8_t* s_t = smem + SM::t_off;
  float* s_sc = reinterpret_cast<float*>(smem + SM::cb_off);
  float* s_mag = s_sc + 16;
  float* s_cf = s_sc + 32;
  float* s_bscale = s_sc + 48;
  uint64_t* bar_p = reinterpret_cast<uint64_t*>(smem + SM::bar_off) + 1;
  uint64_t* bar_m = bar_p + 1;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + SM::tmem_off);

  const int tid = threadIdx.x, warp = tid >> 5;
  const int r = tid & (kRows - 1);  // row in the tile = TMEM lane
  const int h = warp >> 2;          // half of the columns
  const int64_t n = a.n;
  const int64_t ntiles = (n + kRows - 1) / kRows;
  const uint32_t buf_s = smem_u32(smem + SM::buf_off), pi_s = smem_u32(s_pi), t_s = smem_u32(s_t);
  const bool vec = (a.ldc & 1) == 0 && (reinterpret_cast<uintptr_t>(a.codes_in) & 7u) == 0;
  const bool svec = (a.lds & 1) == 0 && (reinterpret_cast<uintptr_t>(a.signs_in) & 7u) == 0;

  if (tid == 0) {
    tma_prefetch_desc(&map_pi);
    tma_prefetch_desc(&map_t);
    tma_prefetch_desc(&map_o);
    mbar_init(bar_p, 1);
    mbar_init(bar_m, 1);
    fence_barrier_init();
  }
  if (warp == 0) tmem_alloc(s_tmem, kNcols);
  build_consts<BITS>(a.centroids, s_sc, s_mag, s_cf, s_bscale);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;
  const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
  const uint32_t tm_z = tmem + lane_off + 64u * (uint32_t)h;            // this half's T^T s, then Pi^T w
  const uint32_t tm_s = tmem + 128u + lane_off + 32u * (uint32_t)h;     // this half's sign operand words
  if (tid == 0) {
    mbar_arrive_expect_tx(bar_p, 2 * kTileBytes);
    for (int b = 0; b < 2; ++b) tma_load_2d(s_pi + b * kBoxBytes, &map_pi, b * 64, 0, bar_p);
    for (int b = 0; b < 2; ++b) tma_load_2d(s_t + b * kBoxBytes, &map_t, b * 64, 0, bar_p);
  }
  // the centroid table of the quantizer's magnitude sequence (b >= 3 codes: the binary search's)
  if constexpr (BITS >= 3) {
    Bisect<BITS> bs;
    bs.magnitudes(s_mag);
    if (tid < H) {
      const float m = bs.mag(tid);
      s_cf[H + tid] = m;
      s_cf[H - 1 - tid] = -m;
    }
  }
  bool ok = __syncthreads_and(mbar_wait(bar_p, 0, a.status));
  uint32_t par_m = 0;
  auto wait_mma = [&]() {
    const bool w = mbar_wait(bar_m, par_m, a.status);
    par_m ^= 1;
    tc_fence_after();
    return w;
  };

  // this thread's half row of tile `t` (zeros past the last row): code words, sign words, norm, gamma
  auto load_half_row = [&](int64_t t, uint32_t (&wc_)[WH], uint32_t (&sw_)[2], float& nrm_, float& gam_) {
#pragma unroll
    for (int w = 0; w < WH; ++w) wc_[w] = 0u;
    sw_[0] = sw_[1] = 0u;
    nrm_ = gam_ = 0.f;
    const int64_t row = t * kRows + r;
    if (t >= ntiles || row >= n) return;
    const uint32_t* src = a.codes_in + row * a.ldc + WH * h;
    if (vec) {
#pragma unroll
      for (int w = 0; w < WH; w += 2) {
        const uint2 v = __ldg(reinterpret_cast<const uint2*>(src + w));
        wc_[w] = v.x, wc_[w + 1] = v.y;
      }
    } else {
#pragma unroll
      for (int w = 0; w < WH; ++w) wc_[w] = __ldg(src + w);
    }
    const uint32_t* ssrc = a.signs_in + row * a.lds + (NS / 2) * h;
    if (svec) {
      const uint2 v = __ldg(reinterpret_cast<const uint2*>(ssrc));
      sw_[0] = v.x, sw_[1] = v.y;
    } else {
      sw_[0] = __ldg(ssrc), sw_[1] = __ldg(ssrc + 1);
    }
    nrm_ = __ldg(a.norms_in + row * a.ldn);
    gam_ = __ldg(a.gammas_in + row * a.ldn);
  };
  uint32_t wc[WH], sw[2];
  float nrm, gam;
  load_half_row(blockIdx.x, wc, sw, nrm, gam);

  for (int64_t tile = blockIdx.x; ok && tile < ntiles; tile += gridDim.x) {
    const int64_t row0 = tile * kRows;
    // the next tile's inputs are loaded while this one is computed
    uint32_t wc_n[WH], sw_n[2];
    float nrm_n, gam_n;
    load_half_row(tile + gridDim.x, wc_n, sw_n, nrm_n, gam_n);
    // +-1 (fp16) sign operand of this half: bit 1 = +1, a pair of coordinates per word
#pragma unroll
    for (int cc = 0; cc < 2; ++cc) {
      uint32_t so[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const uint32_t t2 = sw[cc] >> (2 * i);
        so[i] = 0xBC00BC00u ^ ((t2 & 1u) << 15) ^ ((t2 & 2u) << 30);
      }
      tmem_st16(tm_s + 16u * (uint32_t)cc, so);
    }
    tmem_wait_st();
    if (tid == 0) bulk_wait_read<0>();  // the previous tile's x_hat store has left the tile buffer
    tc_fence_before();
    ok = __syncthreads_and(ok);
    if (!ok) break;
    if (tid == 0) {  // T^T s per row
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk)
        umma_f16_ts(tmem, tmem + 128u + (uint32_t)(8 * kk), umma_desc_sw128(t_s + (uint32_t)(kk * 16 * 128), kBoxBytes, 1024),
                    kIdTT, kk > 0);
      umma_commit(bar_m);
    }
    if (!wait_mma()) ok = false;
    auto code_at = [&](int kl) -> uint32_t {
      const int bit = kl * BITS, word = bit >> 5, sh = bit & 31;
      uint32_t v = wc[word] >> sh;
      if (sh + BITS > 32) v |= wc[word + 1] << (32 - sh);
      return v & ((1u << BITS) - 1u);
    };
    const float qs = a.qjl_scale * gam;  // sqrt(pi/2)/m * gamma
#pragma unroll
    for (int cc = 0; cc < 2; ++cc) {
      float v[32];
      tmem_ld32(tm_z + 32u * (uint32_t)cc, v);
#pragma unroll
      for (int i = 0; i < 32; ++i) v[i] = fmaf(qs, v[i], s_cf[code_at(32 * cc + i)]);
#pragma unroll
      for (int q = 0; q < 4; ++q) sts_v4(buf_s + sw128_chunk(r, 8 * h + 4 * cc + q, kBoxBytes), Elem<T>::pack(&v[8 * q]));
    }
    fence_proxy_async_smem();
    tc_fence_before();
    ok = __syncthreads_and(ok);
    if (!ok) break;
    if (tid == 0) {  // Pi^T w per row
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t akoff = (uint32_t)((kk >> 2) * kBoxBytes + (kk & 3) * 32);
        umma_f16(tmem, umma_desc_sw128(buf_s + akoff, 16, 1024),
                 umma_desc_sw128(pi_s + (uint32_t)(kk * 16 * 128), kBoxBytes, 1024), kIdPiT, kk > 0);
      }
      umma_commit(bar_m);
    }
    if (!wait_mma()) ok = false;
#pragma unroll
    for (int cc = 0; cc < 2; ++cc) {
      float v[32];
      tmem_ld32(tm_z + 32u * (uint32_t)cc, v);
#pragma unroll
      for (int i = 0; i < 32; ++i) v[i] *= nrm;
#pragma unroll
      for (int q = 0; q < 4; ++q) sts_v4(buf_s + sw128_chunk(r, 8 * h + 4 * cc + q, kBoxBytes), Elem<T>::pack(&v[8 * q]));
    }
    fence_proxy_async_smem();
    tc_fence_before();
    ok = __syncthreads_and(ok);
    if (!ok) break;
    if (tid == 0) {
      for (int b = 0; b < 2; ++b)
        tma_store_2d(&map_o, b * 64, (int32_t)row0, smem + SM::buf_off + b * kBoxBytes);
      bulk_commit();
    }
#pragma unroll
    for (int w = 0; w < WH; ++w) wc[w] = wc_n[w];
    sw[0] = sw_n[0], sw[1] = sw_n[1];
    nrm = nrm_n, gam = gam_n;
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

}  // namespace tq

// ============================================================================ launch
template <typename T, int BITS>
static cudaError_t launch_tq_dq_prod_t(const CUtensorMap& mp, const CUtensorMap& mt, const CUtensorMap& mo,
                                       const TqArgs& a, cudaStream_t st, int num_sms) {
  auto kern = tq::tq_dq_prod_kernel<T, BITS>;
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, tq::SmemP::alloc);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  const int64_t ntiles = (a.n + tq::kRows - 1) / tq::kRows;
  const int64_t grid = std::min<int64_t>(ntiles, (int64_t)num_sms * 2);
  kern<<<(unsigned)grid, tq::kThreadsM, tq::SmemP::alloc, st>>>(mp, mt, mo, a);
  return cudaGetLastError();
}

template <typename T, int BITS, int MODE>
static cudaError_t launch_tq_mse_t(const CUtensorMap& mx, const CUtensorMap& mp, const CUtensorMap& mo,
                                   const TqArgs& a, cudaStream_t st, int num_sms) {
  auto kern = tq::tq_mse_kernel<T, BITS, MODE>;
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, tq::SmemM::alloc);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  const int64_t ntiles = (a.n + tq::kRows - 1) / tq::kRows;
  const int64_t grid = std::min<int64_t>(ntiles, (int64_t)num_sms * 2);
  return launch_pdl(kern, (unsigned)grid, tq::kThreadsM, tq::SmemM::alloc, st, mx, mp, mo, a);
}

template <typename T, int MODE>
static cudaError_t tq_mse_by_bits(int bits, const CUtensorMap& mx, const CUtensorMap& mp, const CUtensorMap& mo,
                                  const TqArgs& a, cudaStream_t st, int sms) {
  switch (bits) {
    case 1: return launch_tq_mse_t<T, 1, MODE>(mx, mp, mo, a, st, sms);
    case 2: return launch_tq_mse_t<T, 2, MODE>(mx, mp, mo, a, st, sms);
    case 3: return launch_tq_mse_t<T, 3, MODE>(mx, mp, mo, a, st, sms);
    default: return launch_tq_mse_t<T, 4, MODE>(mx, mp, mo, a, st, sms);
  }
}

template <typename T, int BITS>
static cudaError_t launch_tq_prod_t(const CUtensorMap& mx, const CUtensorMap& mp, const CUtensorMap& mt,
                                    const TqArgs& a, cudaStream_t st, int num_sms) {
  auto kern = tq::tq_prod_kernel<T, BITS>;
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, tq::SmemP::alloc);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  const int64_t ntiles = (a.n + tq::kRows - 1) / tq::kRows;
  const int64_t grid = std::min<int64_t>(ntiles, (int64_t)num_sms * 2);
  return launch_pdl(kern, (unsigned)grid, tq::kThreadsM, tq::SmemP::alloc, st, mx, mp, mt, a);
}

template <typename T>
static cudaError_t tq_prod_by_bits(int bits, const CUtensorMap& mx, const CUtensorMap& mp, const CUtensorMap& mt,
                                   const TqArgs& a, cudaStream_t st, int sms) {
  switch (bits) {
    case 1: return launch_tq_prod_t<T, 1>(mx, mp, mt, a, st, sms);
    case 2: return launch_tq_prod_t<T, 2>(mx, mp, mt, a, st, sms);
    case 3: return launch_tq_prod_t<T, 3>(mx, mp, mt, a, st, sms);
    default: return launch_tq_prod_t<T, 4>(mx, mp, mt, a, st, sms);
  }
}

template <typename T>
static cudaError_t tq_dq_prod_by_bits(int bits, const CUtensorMap& mp, const CUtensorMap& mt, const CUtensorMap& mo,
                                      const TqArgs& a, cudaStream_t st, int sms) {
  switch (bits) {
    case 1: return launch_tq_dq_prod_t<T, 1>(mp, mt, mo, a, st, sms);
    case 2: return launch_tq_dq_prod_t<T, 2>(mp, mt, mo, a, st, sms);
    case 3: return launch_tq_dq_prod_t<T, 3>(mp, mt, mo, a, st, sms);
    default: return launch_tq_dq_prod_t<T, 4>(mp, mt, mo, a, st, sms);
  }
}

template <typename T>
static cudaError_t tq_by_mode(int mode, int bits, const CUtensorMap& mx, const CUtensorMap& mp, const CUtensorMap& mt,
                              const CUtensorMap& mo, const TqArgs& a, cudaStream_t st, int sms) {
  switch (mode) {
    case TQ_MSE_Q: return tq_mse_by_bits<T, TQ_MSE_Q>(bits, mx, mp, mo, a, st, sms);
    case TQ_MSE_QDQ: return tq_mse_by_bits<T, TQ_MSE_QDQ>(bits, mx, mp, mo, a, st, sms);
    case TQ_PROD_Q: return tq_prod_by_bits<T>(bits, mx, mp, mt, a, st, sms);
    case TQ_DQ_MSE: return tq_mse_by_bits<T, TQ_DQ_MSE>(bits, mx, mp, mo, a, st, sms);
    default: return tq_dq_prod_by_bits<T>(bits, mp, mt, mo, a, st, sms);
  }
}

cudaError_t launch_tq(int mode, kvrq_dtype dt, int bits, const CUtensorMap& mx, const CUtensorMap& mp,
                      const CUtensorMap& mt, const CUtensorMap& mo, const TqArgs& a, cudaStream_t st, int sms) {
  if (dt == KVRQ_BF16) return tq_by_mode<__nv_bfloat16>(mode, bits, mx, mp, mt, mo, a, st, sms);
  return tq_by_mode<__half>(mode, bits, mx, mp, mt, mo, a, st, sms);
}

}  // namespace kvrq
