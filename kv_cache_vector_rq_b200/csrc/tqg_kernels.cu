// TurboQuant for any head dimension that is a multiple of 128, and for fp32
// vectors, on tcgen05 tensor cores: a tiled contraction D = A * B with K
// streamed through a ring of shared-memory stages and an epilogue that
// quantizes, sketches or reconstructs.
//
// Method (arXiv 2504.19874 summary page, "方法", Algorithms 1 and 2; "TurboQuant
// 论文解读", "随机旋转（Lemma 1）", "QJL 内积无偏估计（Theorem 2）"), as in the
// d = 128 kernels (tq_kernels.cu): y = Pi u, nearest Lloyd-Max centroid per
// coordinate, x_hat = ||x|| Pi^T c_hat; prod keeps (b-1)-bit codes, the sign
// sketch s = sign(T r_rot) of the rotated residual and gamma = ||r_rot||, and
// reconstructs ||x|| Pi^T (c_hat + sqrt(pi/2)/m gamma T^T s).
//
// Pi (and T) no longer fit in shared memory at large d, so every output tile
// (128 rows x N-tile columns) streams its A rows and B columns over the whole
// K. Every tile therefore sees the whole of its input rows, and takes their
// norms from the chunks it streams: tiles are independent and CTAs walk them
// in (M tile, N tile) order, so concurrently running CTAs share A rows and the
// B slice in L2. The residual of the prod quantizer spans all N tiles of a
// row, so it goes through a caller-provided workspace to a second launch.
//
// Roles (320 threads, one CTA per SM):
//   warps 0-3  epilogue: tcgen05.ld of one accumulator row per thread
//   warps 4-7  either read the x chunks for the norms (fp16/bf16 quantize), or
//              build the A chunks (decoded centroids, +-1 signs, or the fp16
//              hi/lo split of fp32 vectors)
//   warp 8     TMA producer (one lane)
//   warp 9     MMA issuer (one lane); two accumulators in TMEM (2 x N-tile
//              columns) so one tile's epilogue overlaps the next tile's MMAs
//
// fp32 vectors are split x = hi + lo with hi, lo in fp16 after scaling the row
// by a power of two that brings its norm into [1, 2): both halves run through
// the fp16 tensor-core product (two MMAs per K step), which keeps y to about
// 2^-22 of ||x||, far inside the code-boundary margin.

#include <cuda_runtime.h>

#include <type_traits>

#include "kvrq_device.cuh"
#include "tqg_launch.h"

namespace kvrq {
namespace tqg {

constexpr int BM = 128, BK = 64, BN_MAX = 256;
constexpr int kThreads = 320;
constexpr int kSmemLimit = 232448;                // 227 KB per block
constexpr float kShift = 9.313225746154785e-10f;  // 2^-30
constexpr float kSketchScale = 256.0f;

template <typename T>
struct IsBf16 {
  static constexpr bool value = std::is_same<T, __nv_bfloat16>::value;
};
template <typename T>
struct IsF32 {
  static constexpr bool value = std::is_same<T, float>::value;
};

template <typename T, int MODE>
struct Cfg {
  static constexpr bool f32 = IsF32<T>::value;
  static constexpr bool q = MODE == G_MSE_Q || MODE == G_PROD_Q1;          // quantizing epilogue
  static constexpr bool norm_pass = q || MODE == G_SKETCH;                  // per-tile row norms
  static constexpr bool build = MODE == G_DQ_MSE || MODE == G_DQ_PROD1 ||
                                (f32 && (norm_pass || MODE == G_DQ_PROD2));  // warps 4-7 write A
  static constexpr bool split = f32 && MODE != G_PROD_Q2 && MODE != G_DQ_PROD1;
  static constexpr bool readers = !f32 && norm_pass;  // warps 4-7 read x from the A stages
  static constexpr bool out = MODE == G_DQ_MSE || MODE == G_DQ_PROD2;
  static constexpr bool b_mn = MODE == G_DQ_MSE || MODE == G_DQ_PROD1 || MODE == G_DQ_PROD2;
  // operands are bf16 only when the vectors are bf16 and the product is with Pi (or T for a sketch)
  static constexpr bool op_bf16 = IsBf16<T>::value && MODE != G_PROD_Q2 && MODE != G_DQ_PROD1;
  static constexpr int a_bytes = BM * 128 * (split ? 2 : 1);
  static constexpr int b_bytes = BN_MAX * 128;
  static constexpr int stage = a_bytes + b_bytes;
  static constexpr int out_bytes = out ? 2 * BM * 128 : 0;
  static constexpr int S0 = (kSmemLimit - 1024 - out_bytes - 4096) / stage;
  static constexpr int S = S0 > 6 ? 6 : S0;
  static constexpr int outb = S * stage;
  static constexpr int norms = outb + out_bytes;  // [2][BM] norms, [2][BM] row scales
  static constexpr int cb = norms + 4 * BM * 4;   // quantizer constants
  static constexpr int bars = cb + 64 * 4;
  static constexpr int nbars = 3 * S + 9;  // full, empty, aready [S]; acc full/empty, norm full/empty [2]; done
  static constexpr int tmem = bars + nbars * 8;
  static constexpr int alloc = tmem + 16 + 1024;
  static_assert(S >= 2, "pipeline depth");
  static_assert(alloc <= kSmemLimit, "shared memory");
};

// Quantizer constants as in tq_kernels.cu (unit-scale centroids; every step is
// exactly 0 or 1, the chain of centroid differences is rounded step by step).
template <int BITS>
__device__ __forceinline__ void build_consts(const float* __restrict__ c, float* sc, float* mag, float* cf,
                                             float* bscale) {
  constexpr int K = 1 << BITS, H = K / 2;
  const int t = threadIdx.x;
  float tau_min = 1.f;
  if (H > 1) tau_min = 0.5f * (c[H] + c[H + 1]);
  const int e = (int)((__float_as_uint(tau_min) >> 23) & 0xFF) - 127;
  const float B = __uint_as_float((uint32_t)(127 + 48 - e) << 23);
  if (t == 0) *bscale = B;
  if (t < H) mag[t] = c[H + t];
  if (t < H - 1) sc[t] = -(0.5f * (c[H + t] + c[H + 1 + t])) * B;
  if (t == 0) {
    float ch = c[H];
    for (int j = 0; j < H; ++j) {
      if (j > 0) ch = __fadd_rn(ch, __fsub_rn(c[H + j], c[H + j - 1]));
      cf[H + j] = ch;
      cf[H - 1 - j] = -ch;
    }
  }
}

// Barrier among the 128 epilogue threads; returns the AND of `pred` over them.
__device__ __forceinline__ bool epi_sync_and(bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, 1, 128, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(pred ? 1u : 0u)
      : "memory");
  return r != 0;
}

__device__ __forceinline__ void epi_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

// code of coordinate j (0 <= j < 32) from BITS words holding 32 consecutive codes
template <int BITS>
__device__ __forceinline__ uint32_t code_of(const uint32_t* w, int j) {
  const int bit = j * BITS, word = bit >> 5, sh = bit & 31;
  uint32_t v = w[word] >> sh;
  if (sh + BITS > 32) v |= w[word + 1] << (32 - sh);
  return v & ((1u << BITS) - 1u);
}

template <typename T, int BITS, int MODE>
__global__ void __launch_bounds__(kThreads, 1)
    tqg_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
               const __grid_constant__ CUtensorMap map_o, TqgArgs a, int BN) {
  using C = Cfg<T, MODE>;
  constexpr int S = C::S;
  constexpr int K = 1 << BITS, H = K / 2;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float* s_norm = reinterpret_cast<float*>(smem + C::norms);  // [2][BM]
  float* s_scale = s_norm + 2 * BM;                           // [2][BM]
  float* s_sc = reinterpret_cast<float*>(smem + C::cb);
  float* s_mag = s_sc + 16;
  float* s_cf = s_sc + 32;
  float* s_bscale = s_sc + 48;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::bars);
  uint64_t* empty = full + S;
  uint64_t* aready = empty + S;
  uint64_t* accf = aready + S;
  uint64_t* acce = accf + 2;
  uint64_t* nfull = acce + 2;
  uint64_t* nempty = nfull + 2;
  uint64_t* done = nempty + 2;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + C::tmem);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int KT = a.k_total / BK;
  const int NT = a.n_total / BN;
  const int64_t mtiles = (a.n + BM - 1) / BM;
  const int64_t tiles = mtiles * NT;
  const int64_t my_tiles = tiles > (int64_t)blockIdx.x ? (tiles - 1 - blockIdx.x) / gridDim.x + 1 : 0;

  if (tid == 0) {
    if (!C::build) tma_prefetch_desc(&map_a);
    tma_prefetch_desc(&map_b);
    if (C::out) tma_prefetch_desc(&map_o);
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1 + (C::readers ? BM : 0));
      mbar_init(&aready[s], BM);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&accf[b], 1);
      mbar_init(&acce[b], BM);
      mbar_init(&nfull[b], BM);
      mbar_init(&nempty[b], BM);
    }
    mbar_init(done, 1);
    fence_barrier_init();
  }
  if (warp == 0) tmem_alloc(s_tmem, 2 * BN_MAX);
  if (C::q || MODE == G_DQ_MSE || MODE == G_DQ_PROD1) build_consts<BITS>(a.centroids, s_sc, s_mag, s_cf, s_bscale);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;

  if (warp == 8) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      const int64_t a_row0 = (MODE == G_PROD_Q2 || MODE == G_DQ_PROD2) ? 0 : a.map_row0;
      int64_t g = 0;
      bool ok = true;
      for (int64_t i = 0; i < my_tiles && ok; ++i) {
        const int64_t tile = blockIdx.x + i * gridDim.x;
        const int64_t lm = tile / NT;
        const int nt = (int)(tile - lm * NT);
        for (int kc = 0; kc < KT; ++kc) {
          const int s = (int)(g % S);
          const uint32_t ph = (uint32_t)((g / S) & 1);
          if (g >= S && !(ok = mbar_wait(&empty[s], ph ^ 1u, a.status))) break;
          uint8_t* st = smem + s * C::stage;
          mbar_arrive_expect_tx(&full[s], (C::build ? 0u : (uint32_t)C::a_bytes) + (uint32_t)(BN * 128));
          if (!C::build) tma_load_2d(st, &map_a, kc * BK, (int32_t)(a_row0 + lm * BM), &full[s]);
          if (!C::b_mn) {
            tma_load_2d(st + C::a_bytes, &map_b, kc * BK, nt * BN, &full[s]);
          } else {
            for (int q = 0; q < BN / 64; ++q)
              tma_load_2d(st + C::a_bytes + q * (64 * 128), &map_b, nt * BN + q * 64, kc * BK, &full[s]);
          }
          ++g;
        }
      }
      // copies still in flight (only after a failed wait) land before the CTA exits
      for (int64_t j = g > S ? g - S : 0; j < g; ++j) mbar_wait(&full[j % S], (uint32_t)((j / S) & 1), a.status);
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = umma_idesc_f16(C::op_bf16, C::op_bf16, C::b_mn, BN, BM);
      const uint32_t ring_s = smem_u32(smem);
      int64_t g = 0;
      bool ok = true;
      for (int64_t i = 0; i < my_tiles && ok; ++i) {
        const int b = (int)(i & 1);
        if (i >= 2 && !(ok = mbar_wait(&acce[b], (uint32_t)(((i >> 1) - 1) & 1), a.status))) break;
        tc_fence_after();
        const uint32_t d_tm = tmem + (uint32_t)(b * BN);
        for (int kc = 0; kc < KT; ++kc) {
          const int s = (int)(g % S);
          const uint32_t ph = (uint32_t)((g / S) & 1);
          ok = mbar_wait(&full[s], ph, a.status);
          if (ok && C::build) ok = mbar_wait(&aready[s], ph, a.status);
          if (!ok) break;
          tc_fence_after();
          const uint32_t a_s = ring_s + (uint32_t)(s * C::stage), b_s = a_s + C::a_bytes;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint64_t bd = C::b_mn ? umma_desc_sw128(b_s + kk * 2048, 64 * 128, 1024)
                                        : umma_desc_sw128(b_s + kk * 32, 16, 1024);
            umma_f16(d_tm, umma_desc_sw128(a_s + kk * 32, 16, 1024), bd, idesc, kc > 0 || kk > 0);
            if (C::split) umma_f16(d_tm, umma_desc_sw128(a_s + BM * 128 + kk * 32, 16, 1024), bd, idesc, true);
          }
          umma_commit(&empty[s]);
          ++g;
        }
        if (ok) umma_commit(&accf[b]);
      }
      umma_commit(done);  // every MMA issued has completed before TMEM is released
      mbar_wait(done, 0, a.status);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ warps 4-7: norms / A builders
    const int r = tid - 128;
    int64_t g = 0;
    bool ok = true;
    for (int64_t i = 0; i < my_tiles && ok; ++i) {
      const int64_t tile = blockIdx.x + i * gridDim.x;
      const int64_t lm = tile / NT;
      const int b = (int)(i & 1);
      const int64_t lrow = lm * BM + r;
      const bool live = lrow < a.n;
      if constexpr (C::readers) {
        float2 acc[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) acc[k] = make_float2(0.f, 0.f);
        for (int kc = 0; kc < KT; ++kc, ++g) {
          const int s = (int)(g % S);
          if (!(ok = mbar_wait(&full[s], (uint32_t)((g / S) & 1), a.status))) break;
          const uint8_t* st = smem + s * C::stage;
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            float f[8];
            Elem<T>::unpack(*reinterpret_cast<const uint4*>(st + sw128_chunk(r, q, 0)), f);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const float2 v = make_float2(f[2 * k], f[2 * k + 1]);
              acc[k] = __ffma2_rn(v, v, acc[k]);
            }
          }
          // The stage is refilled by TMA (async proxy) once this arrival completes the phase: without the
          // proxy fence, loads still in flight here can return bytes of the next chunk.
          fence_proxy_async_smem();
          mbar_arrive(&empty[s]);
        }
        if (!ok) break;
        if (i >= 2 && !(ok = mbar_wait(&nempty[b], (uint32_t)(((i >> 1) - 1) & 1), a.status))) break;
        s_norm[b * BM + r] =
            sqrtf(((acc[0].x + acc[1].x) + (acc[2].x + acc[3].x)) + ((acc[0].y + acc[1].y) + (acc[2].y + acc[3].y)));
        s_scale[b * BM + r] = 1.f;
        mbar_arrive(&nfull[b]);
      } else if constexpr (C::build) {
        // fp32 rows: norm, and the power-of-two scale that brings it into [1, 2)
        const float* xrow = nullptr;
        float sc = 1.f;
        if constexpr (C::f32 && (C::norm_pass || MODE == G_DQ_PROD2)) {
          xrow = (MODE == G_DQ_PROD2 ? reinterpret_cast<const float*>(a.ws) + lrow * (int64_t)a.d
                                     : a.xf + lrow * a.ldx);
        }
        if constexpr (C::f32 && C::norm_pass) {
          float2 acc[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
          if (live)
            for (int j = 0; j < a.d; j += 4) {
              const float4 v = __ldg(reinterpret_cast<const float4*>(xrow + j));
              acc[0] = __ffma2_rn(make_float2(v.x, v.y), make_float2(v.x, v.y), acc[0]);
              acc[1] = __ffma2_rn(make_float2(v.z, v.w), make_float2(v.z, v.w), acc[1]);
            }
          const float nrm = sqrtf((acc[0].x + acc[1].x) + (acc[0].y + acc[1].y));
          sc = nrm > 0.f ? ldexpf(1.f, -ilogbf(nrm)) : 1.f;
          if (i >= 2 && !(ok = mbar_wait(&nempty[b], (uint32_t)(((i >> 1) - 1) & 1), a.status))) break;
          s_norm[b * BM + r] = nrm;
          s_scale[b * BM + r] = sc;
          mbar_arrive(&nfull[b]);
        }
        const uint32_t* crow = (MODE == G_DQ_MSE) ? a.codes_in + lrow * a.ldc : nullptr;
        const uint32_t* srow = (MODE == G_DQ_PROD1) ? a.signs_in + lrow * a.lds : nullptr;
        for (int kc = 0; kc < KT; ++kc, ++g) {
          const int s = (int)(g % S);
          if (g >= S && !(ok = mbar_wait(&empty[s], (uint32_t)(((g / S) & 1) ^ 1), a.status))) break;
          uint8_t* st = smem + s * C::stage;
          float v[BK];
          if constexpr (MODE == G_DQ_MSE) {
            uint32_t w[2 * BITS];
#pragma unroll
            for (int q = 0; q < 2 * BITS; ++q) w[q] = live ? __ldg(crow + kc * 2 * BITS + q) : 0u;
#pragma unroll
            for (int j = 0; j < BK; ++j) v[j] = s_cf[code_of<BITS>(w + (j >> 5) * BITS, j & 31)];
          } else if constexpr (MODE == G_DQ_PROD1) {
            const uint32_t w0 = live ? __ldg(srow + 2 * kc) : 0u, w1 = live ? __ldg(srow + 2 * kc + 1) : 0u;
#pragma unroll
            for (int j = 0; j < BK; ++j) v[j] = (((j < 32 ? w0 : w1) >> (j & 31)) & 1u) ? 1.f : -1.f;
          } else {
#pragma unroll
            for (int j = 0; j < BK; j += 4) {
              const float4 x4 = live ? __ldg(reinterpret_cast<const float4*>(xrow + kc * BK + j))
                                     : make_float4(0.f, 0.f, 0.f, 0.f);
              v[j] = x4.x * sc;
              v[j + 1] = x4.y * sc;
              v[j + 2] = x4.z * sc;
              v[j + 3] = x4.w * sc;
            }
          }
          if constexpr (C::split) {
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              float hi[8], lo[8];
#pragma unroll
              for (int e = 0; e < 8; ++e) {
                hi[e] = __half2float(__float2half_rn(v[8 * q + e]));
                lo[e] = v[8 * q + e] - hi[e];
              }
              *reinterpret_cast<uint4*>(st + sw128_chunk(r, q, 0)) = Elem<__half>::pack(hi);
              *reinterpret_cast<uint4*>(st + BM * 128 + sw128_chunk(r, q, 0)) = Elem<__half>::pack(lo);
            }
          } else if constexpr (MODE == G_DQ_PROD1) {
#pragma unroll
            for (int q = 0; q < 8; ++q)
              *reinterpret_cast<uint4*>(st + sw128_chunk(r, q, 0)) = Elem<__half>::pack(&v[8 * q]);
          } else {
#pragma unroll
            for (int q = 0; q < 8; ++q)
              *reinterpret_cast<uint4*>(st + sw128_chunk(r, q, 0)) = Elem<T>::pack(&v[8 * q]);
          }
          fence_proxy_async_smem();
          mbar_arrive(&aready[s]);
        }
      }
    }
  } else {
    // ------------------------------------------------------------ warps 0-3: epilogue
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    int64_t nbox = 0;
    bool ok = true;
    for (int64_t i = 0; i < my_tiles; ++i) {
      const int64_t tile = blockIdx.x + i * gridDim.x;
      const int64_t lm = tile / NT;
      const int nt = (int)(tile - lm * NT);
      const int b = (int)(i & 1);
      const uint32_t ph = (uint32_t)((i >> 1) & 1);
      const int64_t lrow = lm * BM + tid;
      const bool live = lrow < a.n;
      const int col0 = nt * BN;
      float nrm = 0.f, sc = 1.f, gam = 0.f;
      if constexpr (C::norm_pass) {
        ok = mbar_wait(&nfull[b], ph, a.status);
        nrm = s_norm[b * BM + tid];
        sc = s_scale[b * BM + tid];
        mbar_arrive(&nempty[b]);
      } else if constexpr (MODE == G_DQ_MSE || MODE == G_DQ_PROD2) {
        nrm = live ? __ldg(a.norms_in + lrow * a.ldn) : 0.f;
      } else if constexpr (MODE == G_DQ_PROD1) {
        gam = live ? __ldg(a.gammas_in + lrow * a.ldn) : 0.f;
      }
      ok = ok && mbar_wait(&accf[b], ph, a.status);
      if (!epi_sync_and(ok)) break;
      tc_fence_after();
      const uint32_t tm = tmem + (uint32_t)(b * BN) + lane_off;

      if constexpr (C::q) {
        const float neff = nrm * sc;  // the accumulator holds Pi (sc x)
        const float srow = neff > 0.f ? __fdiv_rn(*s_bscale, neff) : 0.f;
        const float shift = -fmaf(kShift, neff, 0x1p-126f);
        const float rn = neff > 0.f ? __frcp_rn(neff) : 0.f;
        float dl[H > 1 ? H - 1 : 1], sct[H > 1 ? H - 1 : 1];
#pragma unroll
        for (int j = 0; j < H - 1; ++j) {
          dl[j] = __fsub_rn(s_mag[j + 1], s_mag[j]);
          sct[j] = s_sc[j];
        }
        const float mn0 = s_mag[0];
        uint32_t* crow = a.codes_out + lrow * a.ldc + (col0 / 32) * BITS;
        __half* wrow = reinterpret_cast<__half*>(a.ws) + lrow * (int64_t)a.d + col0;
        float gs = 0.f;
#pragma unroll 1
        for (int c = 0; c < BN / 32; ++c) {
          float y[32];
          tmem_ld32(tm + 32 * c, y);
          uint32_t w[BITS];
#pragma unroll
          for (int q = 0; q < BITS; ++q) w[q] = 0u;
          float rr[32];
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const float Y = y[e] + shift;
            float m = mn0, cnt = 0.5f;
#pragma unroll
            for (int j = 0; j < H - 1; ++j) {
              const float stp = fma_sat(fabsf(Y), srow, sct[j]);
              m = fmaf(stp, dl[j], m);
              cnt += stp;
            }
            const float sg = sign_one(Y);
            const float chat = __fmul_rn(m, sg);
            const uint32_t code = (uint32_t)fmaf(sg, cnt, (float)H - 0.5f);
            const int bit = e * BITS;
            w[bit >> 5] |= code << (bit & 31);
            if ((bit & 31) + BITS > 32) w[(bit >> 5) + 1] |= code >> (32 - (bit & 31));
            if constexpr (MODE == G_PROD_Q1) {
              const float rv = fmaf(y[e], rn, -chat);  // rotated unit residual
              gs = fmaf(rv, rv, gs);
              rr[e] = rv * kSketchScale;
            }
          }
          if (live) {
#pragma unroll
            for (int q = 0; q < BITS; ++q) crow[c * BITS + q] = w[q];
            if constexpr (MODE == G_PROD_Q1) {
#pragma unroll
              for (int q = 0; q < 4; ++q)
                *reinterpret_cast<uint4*>(wrow + 32 * c + 8 * q) = Elem<__half>::pack(&rr[8 * q]);
            }
          }
        }
        if (live) {
          if (nt == 0 && a.norms_out) a.norms_out[lrow * a.ldn] = nrm;
          if constexpr (MODE == G_PROD_Q1) a.part[lrow * a.n_part + nt] = gs;
        }
      } else if constexpr (MODE == G_PROD_Q2 || MODE == G_SKETCH) {
        uint32_t* srow = a.signs_out + lrow * a.lds + col0 / 32;
#pragma unroll 1
        for (int c = 0; c < BN / 32; ++c) {
          float z[32];
          tmem_ld32(tm + 32 * c, z);
          uint32_t bits = 0;
#pragma unroll
          for (int e = 0; e < 32; ++e) bits |= (z[e] >= 0.f ? 1u : 0u) << e;  // sign(0) = +1
          if (live) srow[c] = bits;
        }
        if (live && nt == 0 && a.gammas_out) {
          float gg;
          if constexpr (MODE == G_PROD_Q2) {
            gg = 0.f;
            for (int p = 0; p < a.n_part; ++p) gg += a.part[lrow * a.n_part + p];
            gg = sqrtf(gg);
          } else {
            gg = nrm;
          }
          a.gammas_out[lrow * a.ldn] = gg;
        }
      } else if constexpr (MODE == G_DQ_PROD1) {
        const float qs = a.qjl_scale * gam;
        const uint32_t* crow = a.codes_in + lrow * a.ldc + (col0 / 32) * BITS;
        T* wrow = reinterpret_cast<T*>(a.ws) + lrow * (int64_t)a.d + col0;
        constexpr int PC = Elem<T>::kPerChunk;
#pragma unroll 1
        for (int c = 0; c < BN / 32; ++c) {
          float v[32];
          tmem_ld32(tm + 32 * c, v);
          uint32_t w[BITS];
#pragma unroll
          for (int q = 0; q < BITS; ++q) w[q] = live ? __ldg(crow + c * BITS + q) : 0u;
#pragma unroll
          for (int e = 0; e < 32; ++e) v[e] = fmaf(qs, v[e], s_cf[code_of<BITS>(w, e)]);
          if (live) {
#pragma unroll
            for (int q = 0; q < 32 / PC; ++q)
              *reinterpret_cast<uint4*>(wrow + 32 * c + PC * q) = Elem<T>::pack(&v[PC * q]);
          }
        }
      } else {
        // x_hat = ||x|| * acc, staged through two 128-byte x 128-row boxes, TMA store
        constexpr int PC = Elem<T>::kPerChunk;
        constexpr int kCols = 128 / (int)sizeof(T);  // columns per box
        constexpr int GPB = kCols / 32;              // 32-column groups per box
#pragma unroll 1
        for (int c = 0; c < BN / 32; ++c) {
          if (c % GPB == 0) {
            if (tid == 0) bulk_wait_read<1>();  // the box that last used this buffer has been read
            epi_sync();
          }
          float v[32];
          tmem_ld32(tm + 32 * c, v);
#pragma unroll
          for (int e = 0; e < 32; ++e) v[e] *= nrm;
          uint8_t* buf = smem + C::outb + (int)(nbox & 1) * (BM * 128);
#pragma unroll
          for (int q = 0; q < 32 / PC; ++q)
            *reinterpret_cast<uint4*>(buf + sw128_chunk(tid, (c % GPB) * (32 / PC) + q, 0)) =
                Elem<T>::pack(&v[PC * q]);
          if (c % GPB == GPB - 1) {
            fence_proxy_async_smem();
            epi_sync();
            if (tid == 0) {
              tma_store_2d(&map_o, col0 + (c / GPB) * kCols, (int32_t)(a.map_row0 + lm * BM), buf);
              bulk_commit();
            }
            ++nbox;
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&acce[b]);
    }
    if (C::out && tid == 0) bulk_wait_all<0>();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 2 * BN_MAX);
}

}  // namespace tqg

// ============================================================================ launch
template <typename T, int BITS, int MODE>
static cudaError_t launch_tqg_t(const CUtensorMap& ma, const CUtensorMap& mb, const CUtensorMap& mo, const TqgArgs& a,
                                int bn, cudaStream_t st, int sms) {
  using C = tqg::Cfg<T, MODE>;
  auto kern = tqg::tqg_kernel<T, BITS, MODE>;
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::alloc);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  const int64_t tiles = (a.n + tqg::BM - 1) / tqg::BM * (a.n_total / bn);
  const int64_t grid = tiles < sms ? tiles : sms;
  if (grid <= 0) return cudaSuccess;
  kern<<<(unsigned)grid, tqg::kThreads, C::alloc, st>>>(ma, mb, mo, a, bn);
  return cudaGetLastError();
}

template <typename T, int MODE>
static cudaError_t tqg_by_bits(int bits, const CUtensorMap& ma, const CUtensorMap& mb, const CUtensorMap& mo,
                               const TqgArgs& a, int bn, cudaStream_t st, int sms) {
  switch (bits) {
    case 1: return launch_tqg_t<T, 1, MODE>(ma, mb, mo, a, bn, st, sms);
    case 2: return launch_tqg_t<T, 2, MODE>(ma, mb, mo, a, bn, st, sms);
    case 3: return launch_tqg_t<T, 3, MODE>(ma, mb, mo, a, bn, st, sms);
    default: return launch_tqg_t<T, 4, MODE>(ma, mb, mo, a, bn, st, sms);
  }
}

template <typename T>
static cudaError_t tqg_by_mode(int mode, int bits, const CUtensorMap& ma, const CUtensorMap& mb, const CUtensorMap& mo,
                               const TqgArgs& a, int bn, cudaStream_t st, int sms) {
  switch (mode) {
    case G_MSE_Q: return tqg_by_bits<T, G_MSE_Q>(bits, ma, mb, mo, a, bn, st, sms);
    case G_PROD_Q1: return tqg_by_bits<T, G_PROD_Q1>(bits, ma, mb, mo, a, bn, st, sms);
    case G_PROD_Q2: return launch_tqg_t<T, 1, G_PROD_Q2>(ma, mb, mo, a, bn, st, sms);
    case G_SKETCH: return launch_tqg_t<T, 1, G_SKETCH>(ma, mb, mo, a, bn, st, sms);
    case G_DQ_MSE: return tqg_by_bits<T, G_DQ_MSE>(bits, ma, mb, mo, a, bn, st, sms);
    case G_DQ_PROD1: return tqg_by_bits<T, G_DQ_PROD1>(bits, ma, mb, mo, a, bn, st, sms);
    default: return launch_tqg_t<T, 1, G_DQ_PROD2>(ma, mb, mo, a, bn, st, sms);
  }
}

cudaError_t launch_tqg(int mode, kvrq_dtype dt, int bits, int n_tile, const CUtensorMap& map_a,
                       const CUtensorMap& map_b, const CUtensorMap& map_o, const TqgArgs& a, cudaStream_t st,
                       int num_sms) {
  if (dt == KVRQ_F32) return tqg_by_mode<float>(mode, bits, map_a, map_b, map_o, a, n_tile, st, num_sms);
  if (dt == KVRQ_BF16) return tqg_by_mode<__nv_bfloat16>(mode, bits, map_a, map_b, map_o, a, n_tile, st, num_sms);
  return tqg_by_mode<__half>(mode, bits, map_a, map_b, map_o, a, n_tile, st, num_sms);
}

template <typename T>
static int smem_by_mode(int mode) {
  switch (mode) {
    case G_MSE_Q: return tqg::Cfg<T, G_MSE_Q>::alloc;
    case G_PROD_Q1: return tqg::Cfg<T, G_PROD_Q1>::alloc;
    case G_PROD_Q2: return tqg::Cfg<T, G_PROD_Q2>::alloc;
    case G_SKETCH: return tqg::Cfg<T, G_SKETCH>::alloc;
    case G_DQ_MSE: return tqg::Cfg<T, G_DQ_MSE>::alloc;
    case G_DQ_PROD1: return tqg::Cfg<T, G_DQ_PROD1>::alloc;
    default: return tqg::Cfg<T, G_DQ_PROD2>::alloc;
  }
}

int tqg_smem_bytes(int mode, kvrq_dtype dt, int) {
  if (dt == KVRQ_F32) return smem_by_mode<float>(mode);
  if (dt == KVRQ_BF16) return smem_by_mode<__nv_bfloat16>(mode);
  return smem_by_mode<__half>(mode);
}

}  // namespace kvrq
