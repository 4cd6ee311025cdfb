// RotorQuant quantize / dequantize / fused roundtrip kernels for sm_100a.
//
// Method ("TurboQuant + RotorQuant", sections "How RotorQuant Works",
// "The Fused CUDA Kernel", "Codebook Calibration Fix"): split off the L2 norm,
// cut the vector into groups of 3 (zero-padded to 3G), rotate each group with
// its rotor sandwich v' = R v R~, replace each rotated coordinate by the index
// of its nearest Lloyd-Max centroid, pack the codes; dequantize by the inverse
// sandwich R~ v R, drop the pad, multiply by the norm.
//
// B200 design (not the pages' one-thread-per-(vector, group) layout):
//  * d = 128 rows go through `rq_row_kernel`: one thread owns one whole row, a
//    persistent CTA streams 128-row tiles in with TMA (128-byte swizzle, so a
//    thread reading its own row hits 8 different banks per 16-byte phase),
//    double-buffered on mbarriers; results are written to a swizzled shared
//    tile and leave through a TMA tensor store; codes are staged in shared
//    memory and written out coalesced.
//  * The sandwich is applied as its exact 3x3 matrix (9 FMA per group instead
//    of the 48-FMA sparse product the README counts): the matrix is built once
//    per CTA from the rotors.
//  * Quantization compares |y| with the positive Lloyd-Max boundaries scaled by
//    the row norm (so x is never divided by its norm), exploiting the exact
//    symmetry of the codebook.
//  * Any other d (and unaligned rows) go through `rq_general_kernel`: one warp
//    per row, groups strided over lanes, codes assembled per warp in shared
//    memory.

#include <cuda_runtime.h>

#include "kvrq_device.cuh"
#include "rq_launch.h"

namespace kvrq {

// ----------------------------------------------------------------------------
// Scalar quantizer on a row-scaled codebook.
// Codebook c[0..K) is ascending and exactly symmetric; H = K/2. The positive
// boundaries are tau[j] = (c[H-1+j] + c[H+j]) / 2, j = 1..H-1 (tau_0 = 0).
// For y > 0 the code is H + #{j : |y| > tau_j}, for y <= 0 it is
// H - 1 - #{j : |y| > tau_j}; this is the nearest centroid with ties to the
// lower index except when |y| equals a nonzero boundary exactly. `tn` holds
// tau_j * ||x|| and `mn` holds c[H+j] * ||x||, and y is the unnormalised
// rotated coordinate, so the decision is y/||x|| against the boundaries.
template <int BITS>
struct Quantizer {
  static constexpr int K = 1 << BITS;
  static constexpr int H = K / 2;
  float tn[H > 1 ? H - 1 : 1];
  float mn[H];

  __device__ __forceinline__ void scale(const float* tau, const float* mag, float n) {
#pragma unroll
    for (int j = 0; j < H - 1; ++j) tn[j] = tau[j] * n;
#pragma unroll
    for (int j = 0; j < H; ++j) mn[j] = mag[j] * n;
  }

  // returns the code; chat = scaled centroid (||x|| * c[code])
  __device__ __forceinline__ uint32_t operator()(float y, float& chat) const {
    const float a = fabsf(y);
    uint32_t cnt = 0;
    float m = mn[0];
#pragma unroll
    for (int j = 0; j < H - 1; ++j) {
      const bool p = a > tn[j];
      cnt += p ? 1u : 0u;
      m = p ? mn[j + 1] : m;
    }
    const bool pos = y > 0.f;
    chat = pos ? m : -m;
    return pos ? (uint32_t)H + cnt : (uint32_t)(H - 1) - cnt;
  }
};

// Packs code j (compile-time index) into the register bit stream.
template <int BITS, int W>
__device__ __forceinline__ void put_code(uint32_t (&w)[W], int j, uint32_t code) {
  const int bit = j * BITS;
  const int word = bit >> 5;
  const int sh = bit & 31;
  w[word] |= code << sh;
  if (sh + BITS > 32) w[word + 1] |= code >> (32 - sh);
}

template <int BITS, int W>
__device__ __forceinline__ uint32_t get_code(const uint32_t (&w)[W], int j) {
  const int bit = j * BITS;
  const int word = bit >> 5;
  const int sh = bit & 31;
  uint32_t v = w[word] >> sh;
  if (sh + BITS > 32) v |= w[word + 1] << (32 - sh);
  return v & ((1u << BITS) - 1u);
}

// Rotation matrices (9 floats padded to 12) for all groups, and the codebook
// split into positive boundaries and magnitudes, built by the whole CTA.
__device__ __forceinline__ void build_rotor_table(const float* __restrict__ rotors, int G, float4* __restrict__ mtab) {
  for (int g = threadIdx.x; g < G; g += blockDim.x) {
    const float4 r = __ldg(reinterpret_cast<const float4*>(rotors) + g);
    float m[9];
    rotor_matrix(r.x, r.y, r.z, r.w, m);
    mtab[3 * g + 0] = make_float4(m[0], m[1], m[2], m[3]);
    mtab[3 * g + 1] = make_float4(m[4], m[5], m[6], m[7]);
    mtab[3 * g + 2] = make_float4(m[8], 0.f, 0.f, 0.f);
  }
}

template <int BITS>
__device__ __forceinline__ void build_codebook(const float* __restrict__ centroids, float* tau, float* mag, float* cfull) {
  constexpr int K = 1 << BITS, H = K / 2;
  if (threadIdx.x < H) mag[threadIdx.x] = centroids[H + threadIdx.x];
  if ((int)threadIdx.x < H - 1) tau[threadIdx.x] = 0.5f * (centroids[H + threadIdx.x] + centroids[H + 1 + threadIdx.x]);
  if (cfull && threadIdx.x < K) cfull[threadIdx.x] = centroids[threadIdx.x];
}

// ============================================================================
// d = 128, one thread per row, TMA-streamed 128-row tiles.
// ============================================================================
template <typename T>
struct RowTile {
  static constexpr int D = 128;
  static constexpr int kRows = 128;
  static constexpr int kBoxElems = 128 / sizeof(T);        // elements per 128-byte box row
  static constexpr int kBoxes = D / kBoxElems;             // boxes per tile (2 for 16-bit, 4 for fp32)
  static constexpr int kBoxBytes = kRows * 128;            // 16 KB
  static constexpr int kTileBytes = kBoxes * kBoxBytes;    // 32 KB (16-bit) / 64 KB (fp32)
  static constexpr int kChunks = D * (int)sizeof(T) / 16;  // 16-byte chunks per row
  static constexpr int kE = 16 / (int)sizeof(T);           // elements per chunk
  static constexpr int kStages = 2;

  // byte offset of 16-byte chunk j of row r inside a swizzled tile
  __device__ __forceinline__ static uint32_t chunk_offset(int r, int j) {
    const int box = j >> 3, c = j & 7;
    return (uint32_t)(box * kBoxBytes + r * 128 + ((c ^ (r & 7)) << 4));
  }
};

template <int BITS>
struct RowCodes {
  static constexpr int G = 43;
  static constexpr int NC = 3 * G;
  static constexpr int W = (NC * BITS + 31) / 32;
};

// Shared memory layout of the row kernel (offsets from a 1024-aligned base).
template <typename T, int BITS, int MODE>
struct RowSmem {
  using TL = RowTile<T>;
  static constexpr int W = RowCodes<BITS>::W;
  static constexpr int K = 1 << BITS;
  static constexpr bool kIn = MODE != RQ_DQ;
  static constexpr bool kOut = MODE != RQ_Q;
  static constexpr int in_off = 0;
  static constexpr int in_bytes = kIn ? TL::kStages * TL::kTileBytes : 0;
  static constexpr int out_off = in_off + in_bytes;
  static constexpr int out_bytes = kOut ? TL::kTileBytes : 0;
  static constexpr int codes_off = out_off + out_bytes;
  static constexpr int codes_bytes = TL::kRows * W * 4;
  static constexpr int lut_off = codes_off + ((codes_bytes + 15) / 16) * 16;
  static constexpr int lut_bytes = MODE == RQ_DQ ? K * TL::kRows * 4 : 0;
  static constexpr int mtab_off = lut_off + lut_bytes;
  static constexpr int mtab_bytes = 3 * 43 * 16;
  static constexpr int cb_off = mtab_off + mtab_bytes;
  static constexpr int cb_bytes = 64 * 4;
  static constexpr int bar_off = cb_off + cb_bytes;
  static constexpr int bytes = bar_off + 64;
  static constexpr int alloc = bytes + 1024;  // room to align the base
};

template <typename T, int BITS, int MODE>
__global__ void __launch_bounds__(128) rq_row_kernel(const __grid_constant__ CUtensorMap map_x,
                                                     const __grid_constant__ CUtensorMap map_o, RqArgs a) {
  using TL = RowTile<T>;
  using SM = RowSmem<T, BITS, MODE>;
  constexpr int D = TL::D, G = RowCodes<BITS>::G, W = RowCodes<BITS>::W, K = 1 << BITS;
  constexpr int S = TL::kStages;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* s_in = smem + SM::in_off;
  uint8_t* s_out = smem + SM::out_off;
  uint32_t* s_codes = reinterpret_cast<uint32_t*>(smem + SM::codes_off);
  float* s_lut = reinterpret_cast<float*>(smem + SM::lut_off);
  float4* s_m = reinterpret_cast<float4*>(smem + SM::mtab_off);
  float* s_tau = reinterpret_cast<float*>(smem + SM::cb_off);
  float* s_mag = s_tau + 16;
  float* s_c = s_tau + 32;
  uint64_t* s_bar = reinterpret_cast<uint64_t*>(smem + SM::bar_off);

  const int tid = threadIdx.x;
  const int64_t n = a.n;
  const int64_t ntiles = (n + TL::kRows - 1) / TL::kRows;

  if (tid == 0) {
    if (SM::kIn) tma_prefetch_desc(&map_x);
    if (SM::kOut) tma_prefetch_desc(&map_o);
    for (int s = 0; s < S; ++s) mbar_init(&s_bar[s], 1);
    fence_barrier_init();
  }
  build_rotor_table(a.rotors, G, s_m);
  build_codebook<BITS>(a.centroids, s_tau, s_mag, s_c);
  __syncthreads();

  // loads issued into each stage (thread 0 only); the k-th load of a stage
  // completes that stage barrier's phase with parity k & 1
  uint32_t issued[S];
#pragma unroll
  for (int s = 0; s < S; ++s) issued[s] = 0;
  auto issue_load = [&](int64_t tile, int s) {
    ++issued[s];
    mbar_arrive_expect_tx(&s_bar[s], TL::kTileBytes);
#pragma unroll
    for (int b = 0; b < TL::kBoxes; ++b)
      tma_load_2d(s_in + s * TL::kTileBytes + b * TL::kBoxBytes, &map_x, b * TL::kBoxElems,
                  (int32_t)(tile * TL::kRows), &s_bar[s]);
  };

  if (SM::kIn && tid == 0) {
    for (int s = 0; s < S; ++s) {
      const int64_t tile = blockIdx.x + (int64_t)s * gridDim.x;
      if (tile < ntiles) issue_load(tile, s);
    }
  }

  int it = 0;
  for (int64_t tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++it) {
    const int s = it % S;
    const uint32_t phase = (uint32_t)((it / S) & 1);
    const int64_t row0 = tile * TL::kRows;
    const int rows = (int)(n - row0 < (int64_t)TL::kRows ? n - row0 : (int64_t)TL::kRows);
    const int64_t row = row0 + tid;

    float x[D];
    uint32_t wc[W];
#pragma unroll
    for (int w = 0; w < W; ++w) wc[w] = 0u;
    float nrm = 0.f;

    bool ok = true;
    if constexpr (SM::kIn) {
      ok = mbar_wait(&s_bar[s], phase, a.status);  // a time-out is recorded in the status word
      const uint8_t* sb = s_in + s * TL::kTileBytes;
#pragma unroll
      for (int j = 0; j < TL::kChunks; ++j) {
        const uint4 v = *reinterpret_cast<const uint4*>(sb + TL::chunk_offset(tid, j));
        Elem<T>::unpack(v, &x[j * TL::kE]);
      }
    } else {
      // dequantize: gather this tile's packed codes (coalesced) into shared memory
      for (int i = tid; i < rows * W; i += TL::kRows) {
        const int r = i / W, w = i - r * W;
        s_codes[i] = __ldg(a.codes_in + (row0 + r) * a.ldc + w);
      }
      nrm = tid < rows ? __ldg(a.norms_in + row) : 0.f;
    }

    if (SM::kOut && tid == 0) bulk_wait_read<0>();  // previous x_hat store has left s_out
    if (!__syncthreads_and(ok)) {
      // a load timed out: wait (bounded) for this CTA's other loads before leaving
      if (SM::kIn && tid == 0)
        for (int s2 = 0; s2 < S; ++s2)
          if (issued[s2]) mbar_wait(&s_bar[s2], (issued[s2] - 1) & 1, a.status);
      break;
    }
    if (SM::kIn && tid == 0) {
      const int64_t next = tile + (int64_t)S * gridDim.x;
      if (next < ntiles) issue_load(next, s);
    }

    Quantizer<BITS> q;
    if constexpr (SM::kIn) {
      float acc[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) acc[k] = 0.f;
#pragma unroll
      for (int i = 0; i < D; ++i) acc[i & 7] = fmaf(x[i], x[i], acc[i & 7]);
      const float ss = ((acc[0] + acc[1]) + (acc[2] + acc[3])) + ((acc[4] + acc[5]) + (acc[6] + acc[7]));
      nrm = sqrtf(ss);
      q.scale(s_tau, s_mag, nrm);
    } else {
#pragma unroll
      for (int w = 0; w < W; ++w) wc[w] = s_codes[tid * W + w];
#pragma unroll
      for (int k = 0; k < K; ++k) s_lut[k * TL::kRows + tid] = s_c[k] * nrm;
    }

    float xo[TL::kE];  // the output chunk being assembled
    uint8_t* so = s_out;
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const float4 m0 = s_m[3 * g], m1 = s_m[3 * g + 1], m2 = s_m[3 * g + 2];
      const float m[9] = {m0.x, m0.y, m0.z, m0.w, m1.x, m1.y, m1.z, m1.w, m2.x};
      float c[3];
      if constexpr (SM::kIn) {
        float v[3];
#pragma unroll
        for (int i = 0; i < 3; ++i) v[i] = (3 * g + i < D) ? x[3 * g + i] : 0.f;
#pragma unroll
        for (int i = 0; i < 3; ++i) {
          float y = m[3 * i] * v[0];
          if (3 * g + 1 < D) y = fmaf(m[3 * i + 1], v[1], y);
          if (3 * g + 2 < D) y = fmaf(m[3 * i + 2], v[2], y);
          const uint32_t code = q(y, c[i]);
          put_code<BITS, W>(wc, 3 * g + i, code);
        }
      } else {
#pragma unroll
        for (int i = 0; i < 3; ++i) c[i] = s_lut[get_code<BITS, W>(wc, 3 * g + i) * TL::kRows + tid];
      }
      if constexpr (SM::kOut) {
#pragma unroll
        for (int i = 0; i < 3; ++i) {
          const int e = 3 * g + i;
          if (e < D) {
            // inverse sandwich: column i of M, i.e. row i of M^T
            const float o = fmaf(m[6 + i], c[2], fmaf(m[3 + i], c[1], m[i] * c[0]));
            xo[e % TL::kE] = o;
            if (e % TL::kE == TL::kE - 1) {
              *reinterpret_cast<uint4*>(so + TL::chunk_offset(tid, e / TL::kE)) = Elem<T>::pack(xo);
            }
          }
        }
      }
    }

    if constexpr (SM::kIn) {
#pragma unroll
      for (int w = 0; w < W; ++w) s_codes[tid * W + w] = wc[w];
      if (tid < rows && a.norms_out) a.norms_out[row] = nrm;
    }
    if constexpr (SM::kOut) fence_proxy_async_smem();
    __syncthreads();
    if constexpr (SM::kOut) {
      if (tid == 0) {
#pragma unroll
        for (int b = 0; b < TL::kBoxes; ++b)
          tma_store_2d(&map_o, b * TL::kBoxElems, (int32_t)row0, s_out + b * TL::kBoxBytes);
        bulk_commit();
      }
    }
    if constexpr (SM::kIn) {
      if (a.codes_out) {
        for (int i = tid; i < rows * W; i += TL::kRows) {
          const int r = i / W, w = i - r * W;
          a.codes_out[(row0 + r) * a.ldc + w] = s_codes[i];
        }
      }
    }
  }
  if (SM::kOut && tid == 0) bulk_wait_all<0>();
}

// ============================================================================
// Any d, any stride: one warp per row.
// ============================================================================
template <typename TI, typename TO, int BITS, int MODE>
__global__ void __launch_bounds__(256) rq_general_kernel(RqArgs a) {
  constexpr int K = 1 << BITS;
  constexpr int SEGW = 3 * BITS;  // words holding the codes of 32 groups (96 codes)
  __shared__ float s_tau[16], s_mag[16], s_c[16];
  __shared__ uint32_t s_seg[8][SEGW];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  build_codebook<BITS>(a.centroids, s_tau, s_mag, s_c);
  if (threadIdx.x < 8 * SEGW) (&s_seg[0][0])[threadIdx.x] = 0u;
  __syncthreads();

  const int d = a.d;
  const int G = (d + 2) / 3;
  const int W = (3 * G * BITS + 31) / 32;
  const TI* __restrict__ xin = reinterpret_cast<const TI*>(a.x);
  TO* __restrict__ xo = reinterpret_cast<TO*>(a.xhat);
  const int64_t warps_total = (int64_t)gridDim.x * (blockDim.x >> 5);

  for (int64_t row = (int64_t)blockIdx.x * (blockDim.x >> 5) + warp; row < a.n; row += warps_total) {
    float nrm;
    if constexpr (MODE != RQ_DQ) {
      const TI* xr = xin + row * a.ldx;
      float ss = 0.f;
      for (int i = lane; i < d; i += 32) {
        const float v = Elem<TI>::to_float(xr[i]);
        ss = fmaf(v, v, ss);
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
      nrm = sqrtf(ss);
      if (lane == 0 && a.norms_out) a.norms_out[row] = nrm;
    } else {
      nrm = __ldg(a.norms_in + row);
    }
    Quantizer<BITS> q;
    q.scale(s_tau, s_mag, nrm);

    for (int gbase = 0; gbase < G; gbase += 32) {
      const int g = gbase + lane;
      const bool active = g < G;
      float c[3] = {0.f, 0.f, 0.f};
      float m[9];
      if (active) {
        const float4 r = __ldg(reinterpret_cast<const float4*>(a.rotors) + g);
        rotor_matrix(r.x, r.y, r.z, r.w, m);
      }
      if constexpr (MODE != RQ_DQ) {
        uint32_t bits3 = 0;  // the group's 3 codes, packed LSB first
        if (active) {
          const TI* xr = xin + row * a.ldx;
          float v[3];
#pragma unroll
          for (int i = 0; i < 3; ++i) v[i] = (3 * g + i < d) ? Elem<TI>::to_float(xr[3 * g + i]) : 0.f;
#pragma unroll
          for (int i = 0; i < 3; ++i) {
            const float y = fmaf(m[3 * i + 2], v[2], fmaf(m[3 * i + 1], v[1], m[3 * i] * v[0]));
            bits3 |= q(y, c[i]) << (i * BITS);
          }
          const int bit = lane * 3 * BITS;  // offset inside this 32-group segment
          atomicOr(&s_seg[warp][bit >> 5], bits3 << (bit & 31));
          if ((bit & 31) + 3 * BITS > 32) atomicOr(&s_seg[warp][(bit >> 5) + 1], bits3 >> (32 - (bit & 31)));
        }
        __syncwarp();
        if (a.codes_out && lane < SEGW) {
          const int wi = (gbase / 32) * SEGW + lane;
          if (wi < W) a.codes_out[row * a.ldc + wi] = s_seg[warp][lane];
        }
        __syncwarp();
        if (lane < SEGW) s_seg[warp][lane] = 0u;
        __syncwarp();
      } else if (active) {
        const uint32_t* cr = a.codes_in + row * a.ldc;
#pragma unroll
        for (int i = 0; i < 3; ++i) {
          const int bit = (3 * g + i) * BITS;
          uint32_t v = __ldg(cr + (bit >> 5)) >> (bit & 31);
          if ((bit & 31) + BITS > 32) v |= __ldg(cr + (bit >> 5) + 1) << (32 - (bit & 31));
          c[i] = s_c[v & (K - 1)] * nrm;
        }
      }
      if constexpr (MODE != RQ_Q) {
        if (active) {
          TO* orow = xo + row * a.ldo;
#pragma unroll
          for (int i = 0; i < 3; ++i) {
            if (3 * g + i < d) {
              const float o = fmaf(m[6 + i], c[2], fmaf(m[3 + i], c[1], m[i] * c[0]));
              orow[3 * g + i] = Elem<TO>::from_float(o);
            }
          }
        }
      }
    }
  }
}

// ============================================================================
// Launch helpers (host)
// ============================================================================
template <typename T, int BITS, int MODE>
static cudaError_t launch_row(const CUtensorMap& mx, const CUtensorMap& mo, const RqArgs& a, cudaStream_t st,
                              int num_sms) {
  using SM = RowSmem<T, BITS, MODE>;
  auto kern = rq_row_kernel<T, BITS, MODE>;
  static int blocks_per_sm = -1;
  if (blocks_per_sm < 0) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SM::alloc);
    if (e != cudaSuccess) return e;
    int b = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, kern, 128, SM::alloc);
    if (e != cudaSuccess) return e;
    blocks_per_sm = b < 1 ? 1 : b;
  }
  const int64_t ntiles = (a.n + 127) / 128;
  const int64_t grid = std::min<int64_t>(ntiles, (int64_t)num_sms * blocks_per_sm);
  kern<<<(unsigned)grid, 128, SM::alloc, st>>>(mx, mo, a);
  return cudaGetLastError();
}

template <typename TI, typename TO, int BITS, int MODE>
static cudaError_t launch_general(const RqArgs& a, cudaStream_t st, int num_sms) {
  const int64_t warps = a.n;
  const int64_t blocks = std::min<int64_t>((warps + 7) / 8, (int64_t)num_sms * 8);
  rq_general_kernel<TI, TO, BITS, MODE><<<(unsigned)blocks, 256, 0, st>>>(a);
  return cudaGetLastError();
}

template <typename T, int MODE>
static cudaError_t row_by_bits(int bits, const CUtensorMap& mx, const CUtensorMap& mo, const RqArgs& a,
                               cudaStream_t st, int sms) {
  switch (bits) {
    case 1: return launch_row<T, 1, MODE>(mx, mo, a, st, sms);
    case 2: return launch_row<T, 2, MODE>(mx, mo, a, st, sms);
    case 3: return launch_row<T, 3, MODE>(mx, mo, a, st, sms);
    default: return launch_row<T, 4, MODE>(mx, mo, a, st, sms);
  }
}

template <int MODE>
static cudaError_t row_by_type(kvrq_dtype dt, int bits, const CUtensorMap& mx, const CUtensorMap& mo,
                               const RqArgs& a, cudaStream_t st, int sms) {
  switch (dt) {
    case KVRQ_F32: return row_by_bits<float, MODE>(bits, mx, mo, a, st, sms);
    case KVRQ_F16: return row_by_bits<__half, MODE>(bits, mx, mo, a, st, sms);
    default: return row_by_bits<__nv_bfloat16, MODE>(bits, mx, mo, a, st, sms);
  }
}

cudaError_t launch_rq_row(int mode, kvrq_dtype dt, int bits, const CUtensorMap& mx, const CUtensorMap& mo,
                          const RqArgs& a, cudaStream_t st, int sms) {
  switch (mode) {
    case RQ_Q: return row_by_type<RQ_Q>(dt, bits, mx, mo, a, st, sms);
    case RQ_DQ: return row_by_type<RQ_DQ>(dt, bits, mx, mo, a, st, sms);
    default: return row_by_type<RQ_QDQ>(dt, bits, mx, mo, a, st, sms);
  }
}

size_t rq_row_smem_bytes(int mode, kvrq_dtype dt, int bits) {
#define KVRQ_SM_CASE(T)                                                   \
  switch (bits) {                                                         \
    case 1: return mode == RQ_Q ? RowSmem<T, 1, RQ_Q>::alloc : mode == RQ_DQ ? RowSmem<T, 1, RQ_DQ>::alloc : RowSmem<T, 1, RQ_QDQ>::alloc; \
    case 2: return mode == RQ_Q ? RowSmem<T, 2, RQ_Q>::alloc : mode == RQ_DQ ? RowSmem<T, 2, RQ_DQ>::alloc : RowSmem<T, 2, RQ_QDQ>::alloc; \
    case 3: return mode == RQ_Q ? RowSmem<T, 3, RQ_Q>::alloc : mode == RQ_DQ ? RowSmem<T, 3, RQ_DQ>::alloc : RowSmem<T, 3, RQ_QDQ>::alloc; \
    default: return mode == RQ_Q ? RowSmem<T, 4, RQ_Q>::alloc : mode == RQ_DQ ? RowSmem<T, 4, RQ_DQ>::alloc : RowSmem<T, 4, RQ_QDQ>::alloc; \
  }
  if (dt == KVRQ_F32) { KVRQ_SM_CASE(float) }
  if (dt == KVRQ_F16) { KVRQ_SM_CASE(__half) }
  KVRQ_SM_CASE(__nv_bfloat16)
#undef KVRQ_SM_CASE
}

template <typename TI, typename TO, int MODE>
static cudaError_t gen_by_bits(int bits, const RqArgs& a, cudaStream_t st, int sms) {
  switch (bits) {
    case 1: return launch_general<TI, TO, 1, MODE>(a, st, sms);
    case 2: return launch_general<TI, TO, 2, MODE>(a, st, sms);
    case 3: return launch_general<TI, TO, 3, MODE>(a, st, sms);
    default: return launch_general<TI, TO, 4, MODE>(a, st, sms);
  }
}

cudaError_t launch_rq_general(int mode, kvrq_dtype dti, kvrq_dtype dto, int bits, const RqArgs& a, cudaStream_t st,
                              int sms) {
  // Q: output type unused (input type reused); DQ: input type unused.
  if (mode == RQ_Q) {
    switch (dti) {
      case KVRQ_F32: return gen_by_bits<float, float, RQ_Q>(bits, a, st, sms);
      case KVRQ_F16: return gen_by_bits<__half, __half, RQ_Q>(bits, a, st, sms);
      default: return gen_by_bits<__nv_bfloat16, __nv_bfloat16, RQ_Q>(bits, a, st, sms);
    }
  }
  if (mode == RQ_DQ) {
    switch (dto) {
      case KVRQ_F32: return gen_by_bits<float, float, RQ_DQ>(bits, a, st, sms);
      case KVRQ_F16: return gen_by_bits<__half, __half, RQ_DQ>(bits, a, st, sms);
      default: return gen_by_bits<__nv_bfloat16, __nv_bfloat16, RQ_DQ>(bits, a, st, sms);
    }
  }
  switch (dti) {
    case KVRQ_F32: return gen_by_bits<float, float, RQ_QDQ>(bits, a, st, sms);
    case KVRQ_F16: return gen_by_bits<__half, __half, RQ_QDQ>(bits, a, st, sms);
    default: return gen_by_bits<__nv_bfloat16, __nv_bfloat16, RQ_QDQ>(bits, a, st, sms);
  }
}

}  // namespace kvrq
