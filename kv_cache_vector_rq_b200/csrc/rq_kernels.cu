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
//  * d = 128 rows (and d = 256 rows of 16-bit types) go through `rq_row_kernel`:
//    one thread owns one whole row and every warp is an independent pipeline
//    over 32-row sub-tiles: its own TMA loads (128-byte swizzle, so a lane
//    reading its own row hits 8 different banks per 16-byte phase), mbarriers,
//    x_hat written back in place and stored by TMA, codes staged in shared
//    memory and stored by one bulk copy. Large d = 128 launches stream each
//    warp's sub-tiles through a ring of three half-tile boxes (see Shape).
//  * The sandwich is applied as its exact 3x3 matrix (9 FMA per group instead
//    of the 48-FMA sparse product the README counts): the matrix is built once
//    per CTA from the rotors.
//  * Quantization compares |y| with the positive Lloyd-Max boundaries scaled by
//    the row norm (so x is never divided by its norm), exploiting the exact
//    symmetry of the codebook.
//  * 16-bit rows of d > 256 (a multiple of 8, up to 4,608) go through
//    `rq_run_kernel`: rows streamed into shared memory by bulk copy, a warp per
//    row, each lane a contiguous run of groups on packed f32x2 FMAs.
//  * Other d with 16-byte aligned rows go through `rq_wide_kernel` (rows
//    streamed into shared memory by bulk copy, a warp per row, groups strided
//    over the lanes); anything else through `rq_general_kernel`: one warp per
//    row, groups strided over lanes, codes assembled per warp in shared memory.

#include <cuda_runtime.h>

#include <type_traits>

#include "bisect.cuh"
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

template <int BITS>
__device__ __forceinline__ void build_codebook(const float* __restrict__ centroids, float* tau, float* mag, float* cfull) {
  constexpr int K = 1 << BITS, H = K / 2;
  if (threadIdx.x < H) mag[threadIdx.x] = centroids[H + threadIdx.x];
  if ((int)threadIdx.x < H - 1) tau[threadIdx.x] = 0.5f * (centroids[H + threadIdx.x] + centroids[H + 1 + threadIdx.x]);
  if (cfull && threadIdx.x < K) cfull[threadIdx.x] = centroids[threadIdx.x];
}

// ============================================================================
// d = 128, one thread per row, TMA-streamed 32-row sub-tiles per warp.
//
// Per row: pass 1 reads the row from the swizzled shared tile and forms
// ||x||^2; pass 2 re-reads it a group pair (6 elements) at a time, rotates
// the pair with packed f32x2 FMAs, quantizes,
// inverse-rotates and writes x_hat back into the same shared positions, from
// where a TMA tensor store writes it out.
//
// Quantization (nearest centroid, ties to the lower index) runs on the FMA
// pipe. With u = y/||x|| the rotated unit coordinate and B = 2^62:
//   step_j = sat(|y'| * (B/||x||) - tau_j * B) is exactly 0 or 1 (near a
//            boundary the exact value of that fused multiply-add is 0 or at
//            least tau_j * B * 2^-47 >= 2^48 in magnitude, since every
//            positive boundary at d = 128 exceeds 2^-8), and it equals
//            [|u| > tau_j] up to the rounding of B/||x|| (relative 2^-24);
//   cnt    = sum_j step_j, the number of positive boundaries below |u|;
//   mag    = ||x|| c[H + cnt], accumulated as ||x|| c[H] + sum_j step_j delta_j;
//   sign   = sign bit of y' = y - 2^-30 ||x|| (an exact zero counts as
//            negative, as the tie rule requires; the shift is far inside the
//            1e-5 decision margin);
//   code   = H - 1/2 + sign (cnt + 1/2),  c_hat = sign mag.
// Codes are added, as exact small integers, into float accumulators that
// start at 2^23; the low 23 mantissa bits of each accumulator are a window
// of the packed bit stream.
// ============================================================================
#ifndef KVRQ_ROW_MIN_WARPS
#define KVRQ_ROW_MIN_WARPS 16  // resident warps per SM the register budget is sized for
#endif

namespace row {

// Row dimension (128 or 256): G groups of 3 (the last zero-padded), NP group
// pairs (the last may pair a group with an all-zero one), NC stored codes.
template <int DD>
struct Dims {
  static constexpr int D = DD;
  static constexpr int G = (DD + 2) / 3;  // 43 / 86
  static constexpr int NP = (G + 1) / 2;  // 22 / 43
  static constexpr int NC = 3 * G;        // 129 / 258
};
constexpr int kWR = 32;       // rows per warp sub-tile

// CTA shape. Ring (launches of at least two sub-tiles per warp, 16-bit rows,
// quantize or fused): one CTA per SM of 16 warps (14 at b = 4, whose code words
// leave room for fewer warps' boxes), each warp streaming its sub-tiles through
// a ring of three half-tile boxes, so the next sub-tile's halves load while the
// current one is computed and a box is reloaded as soon as its x_hat store has
// read it. Otherwise two-warp CTAs with one tile per warp, which also spread a
// small launch over the SMs within one CTA of each other.
template <typename T, int BITS, int MODE, bool RING>
struct Shape {
  static_assert(!RING || (MODE != RQ_DQ && sizeof(T) == 2 && BITS <= 4), "ring shape");
  static constexpr bool kRing = RING;
  static constexpr int kWarps = kRing ? (BITS == 4 ? 14 : 16) : 2;
  static constexpr int kRows = 32 * kWarps;  // threads per CTA
};
constexpr float kB = 4611686018427387904.0f;      // 2^62
constexpr float kShift = 9.313225746154785e-10f;  // 2^-30
constexpr float kWindow0 = 8388608.0f;            // 2^23

template <typename T, int D>
struct Tile {
  static constexpr int kBoxElems = 128 / (int)sizeof(T);  // elements per 128-byte box row
  static constexpr int kBoxes = D / kBoxElems;             // 2 (16-bit) or 4 (fp32)
  static constexpr int kBoxBytes = kWR * 128;              // 4 KB
  static constexpr int kTileBytes = kBoxes * kBoxBytes;    // one warp's sub-tile: 8 KB (16-bit) / 16 KB (fp32)
  static constexpr int kE = 16 / (int)sizeof(T);           // elements per 16-byte chunk
  static constexpr int kChunks = D / kE;
  // byte offset of 16-byte chunk j of row r in the 128-byte-swizzled tile
  __device__ __forceinline__ static uint32_t chunk(int r, int j) {
    return (uint32_t)((j >> 3) * kBoxBytes + r * 128 + (((j & 7) ^ (r & 7)) << 4));
  }
};

template <int BITS, int NC>
struct Codes {
  static constexpr int K = 1 << BITS;
  static constexpr int H = K / 2;
  static constexpr int W = (NC * BITS + 31) / 32;
  static constexpr int CPW = 23 / BITS;  // codes per float window
  static constexpr int NWIN = (NC + CPW - 1) / CPW;
};

template <typename T, int BITS, int MODE, bool RING, int DD, int L>
struct Smem {
  using SH = Shape<T, BITS, MODE, RING>;
  using DM = Dims<DD>;
  using TL = Tile<T, DD>;
  static constexpr int NC = L * DM::G;  // stored codes per row
  static constexpr int STAGES = 1;  // tiles per warp outside the ring
  static constexpr int kWarps = SH::kWarps;
  static constexpr int kRows = SH::kRows;
  static constexpr int W = Codes<BITS, NC>::W;
  static constexpr int kRingBoxes = 3;
  // [warp][box] half-tile boxes (ring) or [warp][stage] sub-tiles
  static constexpr int tile_bytes = SH::kRing ? kWarps * kRingBoxes * TL::kBoxBytes : kWarps * STAGES * TL::kTileBytes;
  static constexpr int nbar = SH::kRing ? kRingBoxes : STAGES + 2;  // barriers per warp
  // code words per warp: dequantize [2][kWR][W] (bulk loads, double-buffered); quantize [kWR][W] (one
  // bulk store per sub-tile: before the warp's next sub-tile writes codes, that store has read them)
  static constexpr int codes_off = tile_bytes;
  static constexpr int codes_stage = ((kWR * W * 4 + 15) / 16) * 16;
  static constexpr int codes_bytes = kWarps * codes_stage * (MODE == RQ_DQ ? 2 : 1);
  static constexpr int lut_off = codes_off + codes_bytes;  // dequantize: [K][kRows] floats
  static constexpr int lut_bytes = MODE == RQ_DQ ? Codes<BITS, NC>::K * kRows * 4 : 0;
  static constexpr int mp_off = lut_off + lut_bytes;  // [NP][10] float2
  static constexpr int mp_bytes = DM::NP * 10 * 8;
  static constexpr int cb_off = mp_off + mp_bytes;  // codebook constants
  static constexpr int cb_bytes = 64 * 4;
  static constexpr int bar_off = cb_off + cb_bytes;  // per warp: ring boxes, or STAGES sub-tiles + 2 code stages
  static constexpr int bytes = bar_off + 8 * kWarps * nbar;
  static constexpr int alloc = bytes + 1024;
  static constexpr bool fits = alloc <= 227 * 1024;
};

// mp[p][3i+j] = (M_{2p}[i][j], M_{2p+1}[i][j]) for the exact sandwich matrices;
// an all-zero padding group (43 at d = 128) has a zero matrix.
template <int DD>
__device__ __forceinline__ void build_pair_table(const float* __restrict__ rotors, float2* __restrict__ mp) {
  for (int g = threadIdx.x; g < 2 * Dims<DD>::NP; g += blockDim.x) {
    float m[9];
    if (g < Dims<DD>::G) {
      const float4 r = __ldg(reinterpret_cast<const float4*>(rotors) + g);
      rotor_matrix(r.x, r.y, r.z, r.w, m);
    } else {
#pragma unroll
      for (int k = 0; k < 9; ++k) m[k] = 0.f;
    }
    float* dst = reinterpret_cast<float*>(mp + (g >> 1) * 10) + (g & 1);
#pragma unroll
    for (int k = 0; k < 9; ++k) dst[2 * k] = m[k];
    dst[18] = 0.f;
  }
}

// sc[j] = -tau_{j+1} B (j < H-1), mag[j] = c[H+j], cf[k] = c[k]
template <int BITS>
__device__ __forceinline__ void build_consts(const float* __restrict__ centroids, float* sc, float* mag, float* cf) {
  constexpr int K = 1 << BITS, H = K / 2;
  const int t = threadIdx.x;
  if (t < H) mag[t] = centroids[H + t];
  if (t < H - 1) sc[t] = -(0.5f * (centroids[H + t] + centroids[H + 1 + t])) * kB;
  if (t < K) cf[t] = centroids[t];
}

template <typename T, int BITS, int MODE, bool RING, int DD, int L>
__global__ void __launch_bounds__(Shape<T, BITS, MODE, RING>::kRows,
                                  RING ? 1
                                       : (MODE == RQ_Q ? KVRQ_ROW_MIN_WARPS / 2 : KVRQ_ROW_MIN_WARPS) /
                                             Shape<T, BITS, MODE, RING>::kWarps)
    rq_row_kernel(const __grid_constant__ CUtensorMap map_x,
                                                       const __grid_constant__ CUtensorMap map_o, RqArgs a) {
  using DM = Dims<DD>;
  // L codes per group: 3 (the vector part) or 4 (the pages' four-grade layout: the vector part and
  // the trivector part, which is identically zero for a unit rotor and stored as the code of 0)
  static_assert(L == 3 || (L == 4 && DD == 128), "codes per group");
  constexpr int D = DM::D, G = DM::G, NP = DM::NP, NC = L * G;
  constexpr int PC = 2 * L;  // codes per group pair
  static_assert(!RING || DD == 128, "the ring holds half-tiles of d = 128 rows");
  using TL = Tile<T, DD>;
  using CD = Codes<BITS, NC>;
  using SM = Smem<T, BITS, MODE, RING, DD, L>;
  static_assert(SM::fits, "shared memory");
  using SH = Shape<T, BITS, MODE, RING>;
  constexpr int STAGES = SM::STAGES;
  constexpr bool kRing = SH::kRing;
  constexpr int kWarps = SH::kWarps, kRows = SH::kRows;
  constexpr int kNB = SM::nbar;  // barriers per warp
  constexpr int H = CD::H, W = CD::W, CPW = CD::CPW, NWIN = CD::NWIN;
  constexpr int E = TL::kE;
  constexpr bool kIn = MODE != RQ_DQ;
  constexpr bool kOut = MODE != RQ_Q;
  constexpr bool kScale = !std::is_same<T, __half>::value;  // fp16 norms always lie in [2^-24, 2^20]

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint32_t* s_codes = reinterpret_cast<uint32_t*>(smem + SM::codes_off);
  float* s_lut = reinterpret_cast<float*>(smem + SM::lut_off);
  const uint32_t mp_a = smem_u32(smem + SM::mp_off);  // the group pairs' sandwich matrices
  float* s_sc = reinterpret_cast<float*>(smem + SM::cb_off);
  float* s_mag = s_sc + 16;
  float* s_cf = s_sc + 32;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // each warp streams its own 32-row sub-tiles: its buffers, barriers and copies
  // barriers: ring [b] boxes; otherwise [s] tiles, [STAGES + c] codes
  uint64_t* w_bar = reinterpret_cast<uint64_t*>(smem + SM::bar_off) + warp * kNB;
  uint8_t* w_tiles = smem + warp * (kRing ? SM::kRingBoxes * TL::kBoxBytes : STAGES * TL::kTileBytes);
  uint32_t* w_codes = s_codes + warp * (MODE == RQ_DQ ? 2 : 1) * (SM::codes_stage / 4);
  const int64_t n = a.n;
  const int nsub = (int)((n + kWR - 1) / kWR);  // n < 2^31 (checked on the host)
  const int gw = (int)blockIdx.x * kWarps + warp, tw = (int)gridDim.x * kWarps;
  // dequantize: a full sub-tile of packed codes is one contiguous, 16-byte aligned block
  const bool codes_bulk = !kIn && a.ldc == W && (reinterpret_cast<uintptr_t>(a.codes_in) & 15) == 0;

  // bit b of `par`: parity of the next phase of barrier b (all lanes);
  // bit b of `pend`: a copy completing on barrier b is in flight (lane 0)
  uint32_t par = 0, pend = 0;

  // ring: CTA c takes sub-tiles c, c + grid, ... (warp-major), so a small launch reaches every SM;
  // otherwise warp gw takes gw, gw + tw, ...
  auto sub_of = [&](int iter) -> int {
    return kRing ? (int)blockIdx.x + (int)gridDim.x * (warp + kWarps * iter) : gw + iter * tw;
  };
  auto issue_box = [&](int sub, int half, int bx) {  // lane 0: half `half` of sub-tile `sub` into ring box bx
    pend |= 1u << bx;
    mbar_arrive_expect_tx(&w_bar[bx], TL::kBoxBytes);
    tma_load_2d(w_tiles + bx * TL::kBoxBytes, &map_x, half * TL::kBoxElems, sub * kWR, &w_bar[bx]);
  };
  auto issue_tile = [&](int sub, int s) {  // lane 0
    pend |= 1u << s;
    mbar_arrive_expect_tx(&w_bar[s], TL::kTileBytes);
#pragma unroll
    for (int b = 0; b < TL::kBoxes; ++b)
      tma_load_2d(w_tiles + s * TL::kTileBytes + b * TL::kBoxBytes, &map_x, b * TL::kBoxElems, sub * kWR,
                  &w_bar[s]);
  };
  auto codes_bulk_tile = [&](int sub) { return codes_bulk && (int64_t)(sub + 1) * kWR <= n; };
  auto issue_codes = [&](int sub, int c) {  // lane 0
    pend |= 1u << (STAGES + c);
    mbar_arrive_expect_tx(&w_bar[STAGES + c], kWR * W * 4);
    bulk_load(w_codes + c * (SM::codes_stage / 4), a.codes_in + (int64_t)sub * kWR * W, kWR * W * 4,
              &w_bar[STAGES + c]);
  };

  // Launched with programmatic stream serialization: the CTA may be resident before the previous
  // kernel of the stream has finished; every global access below follows this wait.
  grid_dep_wait();
  grid_dep_launch();
  // Each warp sets up its own barriers and starts its first copies before the
  // CTA forms its tables, so the rotor loads overlap the first sub-tile's copy.
  if (lane == 0) {
    if (kIn) tma_prefetch_desc(&map_x);
    if (kOut) tma_prefetch_desc(&map_o);
    for (int b = 0; b < kNB; ++b) mbar_init(&w_bar[b], 1);
    fence_barrier_init();
    if constexpr (kRing) {  // sub-tile 0 in boxes 0 and 1, the first half of sub-tile 1 in box 2
      if (sub_of(0) < nsub) {
        issue_box(sub_of(0), 0, 0);
        issue_box(sub_of(0), 1, 1);
      }
      if (sub_of(1) < nsub) issue_box(sub_of(1), 0, 2);
    } else if (kIn) {
      for (int s = 0; s < STAGES; ++s)
        if (sub_of(s) < nsub) issue_tile(sub_of(s), s);
    } else {
      for (int c = 0; c < 2; ++c)
        if (sub_of(c) < nsub && codes_bulk_tile(sub_of(c))) issue_codes(sub_of(c), c);
    }
  }
  build_pair_table<DD>(a.rotors, reinterpret_cast<float2*>(smem + SM::mp_off));
  build_consts<BITS>(a.centroids, s_sc, s_mag, s_cf);
  __syncthreads();

  // dequantize: this lane's norm of sub-tile `sub`, loaded one sub-tile ahead (0 past the last row)
  auto load_norm = [&](int sub) -> float {
    const int64_t rw = (int64_t)sub * kWR + lane;
    return (sub < nsub && rw < n) ? __ldg(a.norms_in + rw * a.ldn) : 0.f;
  };
  float nrm_pf = 0.f;
  if constexpr (!kIn) nrm_pf = load_norm(sub_of(0));

  int it = 0;
  for (int sub = sub_of(0); sub < nsub; sub = sub_of(++it)) {
    const int s = it % STAGES;
    const int cs = it & 1;
    const int64_t row0 = (int64_t)sub * kWR;
    const int rows = (int)(n - row0 < (int64_t)kWR ? n - row0 : (int64_t)kWR);
    const int64_t row = row0 + lane;
    uint8_t* tb = w_tiles + s * TL::kTileBytes;
    // ring: this sub-tile's halves sit in boxes blo (columns 0..63) and bhi (64..127)
    const int blo = (2 * it) % 3, bhi = (2 * it + 1) % 3;
    uint8_t* const box_lo = kRing ? w_tiles + blo * TL::kBoxBytes : tb;
    uint8_t* const box_hi = kRing ? w_tiles + bhi * TL::kBoxBytes : tb + TL::kBoxBytes;
    // shared-window address of 16-byte chunk j of this lane's row (32-bit: see lds_v4)
    const uint32_t lo_a = smem_u32(box_lo), hi_a = smem_u32(box_hi), tb_a = smem_u32(tb);
    auto cptr = [&](int j) -> uint32_t {
      if constexpr (kRing) return ((j >> 3) ? hi_a : lo_a) + (uint32_t)(lane * 128 + (((j & 7) ^ (lane & 7)) << 4));
      else return tb_a + TL::chunk(lane, j);
    };
    uint32_t* stage_codes = w_codes + (kIn ? 0 : cs * (SM::codes_stage / 4));
    const uint32_t stage_a = smem_u32(stage_codes) + (uint32_t)(lane * W * 4);  // this lane's staged words

    // ---------------------------------------------------------------- inputs
    bool ok = true;
    if constexpr (kRing) {
      ok = mbar_wait(&w_bar[blo], (par >> blo) & 1, a.status);
      if (ok) {
        par ^= 1u << blo;
        pend &= ~(1u << blo);
        ok = mbar_wait(&w_bar[bhi], (par >> bhi) & 1, a.status);
        if (ok) {
          par ^= 1u << bhi;
          pend &= ~(1u << bhi);
        }
      }
    } else if constexpr (kIn) {
      // quantize-only: the last sub-tile's codes store has read the staging words (the fused mode
      // waited for its stores before loading this sub-tile)
      if (!kOut && lane == 0) bulk_wait_read<0>();
      ok = mbar_wait(&w_bar[s], (par >> s) & 1, a.status);
      par ^= 1u << s;
      pend &= ~(1u << s);
    } else {
      if (codes_bulk_tile(sub)) {
        ok = mbar_wait(&w_bar[STAGES + cs], (par >> (STAGES + cs)) & 1, a.status);
        par ^= 1u << (STAGES + cs);
        pend &= ~(1u << (STAGES + cs));
      } else {
        for (int i = lane; i < rows * W; i += kWR) {
          const int r = i / W, w = i - r * W;
          stage_codes[i] = __ldg(a.codes_in + (row0 + r) * a.ldc + w);
        }
      }
      if (lane == 0) bulk_wait_read<0>();  // earlier x_hat stores have left the sub-tile buffer
    }
    __syncwarp();
    if (!__all_sync(0xffffffffu, ok)) {
      // a wait ran out: wait (bounded) for this warp's other copies, then leave
      if (lane == 0)
        for (int b = 0; b < kNB; ++b)
          if ((pend >> b) & 1) mbar_wait(&w_bar[b], (par >> b) & 1, a.status);
      break;
    }

    // ---------------------------------------------------------------- per-row scale
    float xs = 1.f;  // power-of-two prescale of the row (fp32 / bf16 rows of extreme norm only)
    float nrm, nq;   // ||x|| and ||xs x||
    uint32_t wc[W];
    if constexpr (kIn) {
      float2 acc[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) acc[k] = make_float2(0.f, 0.f);
#pragma unroll
      for (int j = 0; j < TL::kChunks; ++j) {
        if constexpr (std::is_same<T, __half>::value) {
          // fp16 squares straight into the fp32 sums (the same roundings as converting first)
          const uint4 c = lds_v4(cptr(j));
          const uint32_t cw[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
          for (int k = 0; k < 4; ++k) sq_acc_f16x2(cw[k], acc[(j * 4 + k) & 3].x, acc[(j * 4 + k) & 3].y);
        } else {
          float f[E];
          Elem<T>::unpack(lds_v4(cptr(j)), f);
#pragma unroll
          for (int k = 0; k < E / 2; ++k) {
            const float2 v = make_float2(f[2 * k], f[2 * k + 1]);
            acc[(j * (E / 2) + k) & 3] = __ffma2_rn(v, v, acc[(j * (E / 2) + k) & 3]);
          }
        }
      }
      float ss = ((acc[0].x + acc[1].x) + (acc[2].x + acc[3].x)) + ((acc[0].y + acc[1].y) + (acc[2].y + acc[3].y));
      if (kScale && !(ss >= 0x1p-100f && ss <= 0x1p100f)) {
        xs = ss < 1.f ? 0x1p100f : 0x1p-100f;
        ss = 0.f;
#pragma unroll 1
        for (int j = 0; j < TL::kChunks; ++j) {
          float f[E];
          Elem<T>::unpack(lds_v4(cptr(j)), f);
          for (int k = 0; k < E; ++k) ss = fmaf(f[k] * xs, f[k] * xs, ss);
        }
      }
      nq = sqrtf(ss);
      nrm = kScale ? nq / xs : nq;
      if constexpr (kRing) {
        // the previous sub-tile's stores have read their buffers: the box they left takes the next
        // sub-tile's first half, and the code words can be staged again
        if (lane == 0) {
          bulk_wait_read<0>();
          if (it > 0 && sub_of(it + 1) < nsub) issue_box(sub_of(it + 1), 0, (2 * it + 2) % 3);
        }
        __syncwarp();
      }
    } else {
      nrm = nrm_pf;  // (0 for lanes past the last row)
      nrm_pf = load_norm(sub_of(it + 1));
      nq = nrm;
#pragma unroll
      for (int w = 0; w < W; ++w) wc[w] = stage_codes[lane * W + w];
    }

    // scaled magnitudes as a chain: chain(0) = mag_0 ||x||, chain(j) = chain(j-1) + delta_j
    // (explicitly rounded products and differences: never contracted, so the
    // fused and the dequantize-only kernels build bit-identical chains)
    constexpr bool kBisect = BITS >= 3;
    const float mn0 = __fmul_rn(s_mag[0], nrm);
    float dl[H > 1 ? H - 1 : 1];
    Bisect<kBisect ? BITS : 3> bs;
    if constexpr (kBisect) {
      float Mj[H];
#pragma unroll
      for (int j = 0; j < H; ++j) Mj[j] = __fmul_rn(s_mag[j], nrm);
      bs.magnitudes(Mj);
    } else {
      float prev = mn0;
#pragma unroll
      for (int j = 1; j < H; ++j) {
        const float cur = __fmul_rn(s_mag[j], nrm);
        dl[j - 1] = __fsub_rn(cur, prev);
        prev = cur;
      }
    }
    if constexpr (!kIn) {
      float ch = mn0;
#pragma unroll
      for (int j = 0; j < H; ++j) {
        if constexpr (kBisect) {
          ch = bs.mag(j);
        } else if (j > 0) {
          ch = __fadd_rn(ch, dl[j - 1]);
        }
        s_lut[(H + j) * kRows + tid] = ch;
        s_lut[(H - 1 - j) * kRows + tid] = -ch;
      }
    }
    const uint32_t lut_a = smem_u32(s_lut) + (uint32_t)(tid * 4);  // this thread's column of the table
    const float srow = nq > 0.f ? __fdiv_rn(kB, nq) : 0.f;
    // y' = y - (2^-30 ||x|| + 2^-126): an exact zero (also of a zero row) becomes negative
    const float shv = -fmaf(kShift, nq, 0x1p-126f);
    const float2 shift2 = make_float2(shv, shv);
    float sc[H > 1 ? H - 1 : 1];
#pragma unroll
    for (int j = 0; j < H - 1; ++j) sc[j] = s_sc[j];
    if constexpr (kBisect) bs.thresholds(sc);

    float win[NWIN];
#pragma unroll
    for (int w = 0; w < NWIN; ++w) win[w] = kWindow0;
    if constexpr (L == 4) {
      // trivector codes: the code of exactly 0, H - 1 by the tie rule (integers < 2^23: exact sums)
#pragma unroll
      for (int g = 0; g < G; ++g) {
        win[(4 * g + 3) / CPW] += (float)((H - 1) << (BITS * ((4 * g + 3) % CPW)));
      }
    }
    if constexpr (kIn) {
#pragma unroll
      for (int w = 0; w < W; ++w) wc[w] = 0u;
    }

    // ---------------------------------------------------------------- pass 2
    // One group pair (6 elements) at a time; a 16-byte chunk is read when the
    // pair holding its first element comes up and written back after the pair
    // holding its last element.
    float xe[D + 6], xo[D];
#pragma unroll
    for (int p = 0; p < NP; ++p) {
      if constexpr (kIn) {
#pragma unroll
        for (int e = 6 * p; e < 6 * p + 6; ++e) {
          if (e < D && e % E == 0) {
            Elem<T>::unpack(lds_v4(cptr(e / E)), &xe[e]);
            if constexpr (kScale) {
#pragma unroll
              for (int k = 0; k < E; ++k) xe[e + k] *= xs;
            }
          }
          if (e >= D) xe[e] = 0.f;
        }
      }
      float2 M[10];
#pragma unroll
      for (int q = 0; q < 5; ++q) {
        const uint4 t = lds_v4(mp_a + (uint32_t)((p * 5 + q) * 16));
        M[2 * q] = make_float2(__uint_as_float(t.x), __uint_as_float(t.y));
        M[2 * q + 1] = make_float2(__uint_as_float(t.z), __uint_as_float(t.w));
      }
      float2 C[3];
      if constexpr (kIn) {
        float2 V[3];
#pragma unroll
        for (int j = 0; j < 3; ++j) V[j] = make_float2(xe[6 * p + j], xe[6 * p + 3 + j]);
#pragma unroll
        for (int i = 0; i < 3; ++i) {
          const float2 Y = __ffma2_rn(M[3 * i + 2], V[2], __ffma2_rn(M[3 * i + 1], V[1], __ffma2_rn(M[3 * i], V[0], shift2)));
          float2 m2 = make_float2(mn0, mn0);
          float2 cnt = make_float2(0.5f, 0.5f);
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
          C[i] = __fmul2_rn(m2, sg);
          const float2 code = __ffma2_rn(sg, cnt, make_float2(H - 0.5f, H - 0.5f));
          // codes of group 2p (lane x) and 2p + 1 (lane y) into their windows
          const int kx = L * (2 * p) + i, ky = L * (2 * p + 1) + i;
          win[kx / CPW] = fmaf(code.x, (float)(1u << (BITS * (kx % CPW))), win[kx / CPW]);
          if (2 * p + 1 < G) win[ky / CPW] = fmaf(code.y, (float)(1u << (BITS * (ky % CPW))), win[ky / CPW]);
        }
        // windows whose codes are all in, and the words they complete, leave the registers now
        const int done = PC * (p + 1) < NC ? PC * (p + 1) : NC;  // codes 0 .. done-1 are packed
#pragma unroll
        for (int w = 0; w < NWIN; ++w) {
          const int last = (w + 1) * CPW < NC ? (w + 1) * CPW : NC;  // one past the window's last code
          if (last <= done && last > PC * p) {
            const uint32_t v = __float_as_uint(win[w]) & 0x7fffffu;
            const int bo = w * CPW * BITS;
            wc[bo >> 5] |= v << (bo & 31);
            if ((bo & 31) + CPW * BITS > 32 && (bo >> 5) + 1 < W) wc[(bo >> 5) + 1] |= v >> (32 - (bo & 31));
          }
        }
#pragma unroll
        for (int wi = 0; wi < W; ++wi) {
          // word wi is final once every code overlapping it is packed
          const int last_code = ((32 * wi + 31) / BITS) < NC ? (32 * wi + 31) / BITS : NC - 1;
          const int win_end = ((last_code / CPW) + 1) * CPW < NC ? ((last_code / CPW) + 1) * CPW : NC;
          const int prev_done = PC * p < NC ? PC * p : NC;
          if (win_end <= done && win_end > prev_done) sts_u32(stage_a + (uint32_t)(wi * 4), wc[wi]);
        }
      } else {
#pragma unroll
        for (int i = 0; i < 3; ++i) {
          const int kx = L * (2 * p) + i, ky = L * (2 * p + 1) + i;
          const float cx = __uint_as_float(lds_u32(lut_a + get_code<BITS, W>(wc, kx) * (kRows * 4)));
          const float cy =
              (2 * p + 1 < G) ? __uint_as_float(lds_u32(lut_a + get_code<BITS, W>(wc, ky) * (kRows * 4))) : 0.f;
          C[i] = make_float2(cx, cy);
        }
      }
      if constexpr (kOut) {
#pragma unroll
        for (int i = 0; i < 3; ++i) {
          const float2 X = __ffma2_rn(M[6 + i], C[2], __ffma2_rn(M[3 + i], C[1], __fmul2_rn(M[i], C[0])));
          if (6 * p + i < D) xo[6 * p + i] = X.x;
          if (6 * p + 3 + i < D) xo[6 * p + 3 + i] = X.y;
        }
#pragma unroll
        for (int e = 6 * p; e < 6 * p + 6; ++e)
          if (e < D && e % E == E - 1)
            sts_v4(cptr(e / E), Elem<T>::pack(&xo[e - (E - 1)]));
      }
      if constexpr (kRing) {
        // pair 10 writes the last x_hat chunk of columns 0..63 (pair 9 read their last input chunk):
        // that half leaves now, and once the store has read its box the box takes the next
        // sub-tile's second half
        static_assert(6 * 10 <= 63 && 6 * 10 + 5 >= 63 && 6 * 9 <= 56 && 6 * 9 + 5 >= 56, "half boundary");
        if (p == 10) {
          fence_proxy_async_smem();
          __syncwarp();
          if (kOut && lane == 0) {
            tma_store_2d(&map_o, 0, (int32_t)row0, box_lo);
            bulk_commit();
          }
        }
        if (p == 14 && lane == 0 && sub_of(it + 1) < nsub) {
          if (kOut) bulk_wait_read<0>();
          issue_box(sub_of(it + 1), 1, blo);
        }
      } else if constexpr (kOut) {
        // every box but the last leaves as soon as the pair writing its last x_hat chunk is done
        // (the pairs before it have read its input chunks), so its store overlaps the rest
#pragma unroll
        for (int b = 0; b + 1 < TL::kBoxes; ++b)
          if (p == ((b + 1) * TL::kBoxElems - 1) / 6) {
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              tma_store_2d(&map_o, b * TL::kBoxElems, (int32_t)row0, tb + b * TL::kBoxBytes);
              bulk_commit();
            }
          }
      }
    }

    // ---------------------------------------------------------------- outputs
    if constexpr (kIn) {
      if (lane < rows && a.norms_out) a.norms_out[(a.out_rows ? a.out_rows[row] : row) * a.ldn] = nrm;
    }
    // a full sub-tile of codes leaves as one bulk copy when code rows are contiguous
    const bool codes_bulk_out = kIn && a.codes_out && !a.out_rows && rows == kWR && a.ldc == W &&
                                (reinterpret_cast<uintptr_t>(a.codes_out) & 15) == 0;
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      if constexpr (kOut && kRing) {
        tma_store_2d(&map_o, TL::kBoxElems, (int32_t)row0, box_hi);
      } else if constexpr (kOut) {
        constexpr int b = TL::kBoxes - 1;  // the others left during pass 2
        tma_store_2d(&map_o, b * TL::kBoxElems, (int32_t)row0, tb + b * TL::kBoxBytes);
      }
      if (codes_bulk_out) bulk_store(a.codes_out + row0 * W, stage_codes, kWR * W * 4);
      if (kOut || codes_bulk_out) bulk_commit();
      if constexpr (kRing) {
        // the ring's boxes are refilled at the next sub-tile's norm pass and its pair 14
      } else if constexpr (kIn) {
        const int next = sub_of(it + STAGES);
        if (next < nsub) {
          if (kOut) bulk_wait_read<0>();  // the x_hat store has read this buffer
          issue_tile(next, s);
        }
      } else {
        const int next = sub_of(it + 2);
        if (next < nsub && codes_bulk_tile(next)) issue_codes(next, cs);
      }
    }
    if constexpr (kIn) {
      if (a.codes_out && !codes_bulk_out)
        for (int i = lane; i < rows * W; i += kWR) {
          const int r = i / W, w = i - r * W;
          a.codes_out[(a.out_rows ? a.out_rows[row0 + r] : row0 + r) * a.ldc + w] = stage_codes[i];
        }
    }
  }
  // the stores have read their shared-memory sources; their writes complete with the grid
  if (lane == 0) bulk_wait_read<0>();
}

}  // namespace row

using row::rq_row_kernel;



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
      if (lane == 0 && a.norms_out) a.norms_out[row * a.ldn] = nrm;
    } else {
      nrm = __ldg(a.norms_in + row * a.ldn);
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
// Any d with 16-byte aligned rows (d x element size a multiple of 16): rows
// streamed by bulk copy, processed by a team of TEAM warps per row.
//
// The CTA (8 warps) builds the groups' exact 3x3 sandwich matrices once. A team
// -- one warp for narrow rows, the whole CTA for wide ones (d >= 768) -- owns
// two shared row buffers and bulk-copies blocks of rows into them, so the next
// block is on its way while the current one is processed. Per row the norm is
// a reduction over 16-byte chunks, thread t of the team takes groups t, t +
// team size, ...; a group's codes are OR-ed into the team's word buffer and
// stored coalesced; x_hat overwrites the row in the buffer and the block leaves
// by bulk copy. The quantizer and the reconstruction are those of
// rq_general_kernel, so quantize-then-dequantize and the fused launch agree bit
// for bit.
// ============================================================================
// one element of a row buffer at a 32-bit shared address, as float
template <typename TB>
__device__ __forceinline__ float lds_elem(uint32_t addr) {
  if constexpr (std::is_same<TB, float>::value) {
    return __uint_as_float(lds_u32(addr));
  } else {
    unsigned short v;
    asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(addr));
    if constexpr (std::is_same<TB, __half>::value) return __half2float(__ushort_as_half(v));
    else return __bfloat162float(__ushort_as_bfloat16(v));
  }
}
template <typename TB>
__device__ __forceinline__ void sts_elem(uint32_t addr, float f) {
  if constexpr (std::is_same<TB, float>::value) {
    asm volatile("st.shared.f32 [%0], %1;" ::"r"(addr), "f"(f) : "memory");
  } else {
    const TB h = Elem<TB>::from_float(f);
    unsigned short v;
    if constexpr (std::is_same<TB, __half>::value) v = __half_as_ushort(h);
    else v = __bfloat16_as_ushort(h);
    asm volatile("st.shared.u16 [%0], %1;" ::"r"(addr), "h"(v) : "memory");
  }
}
__device__ __forceinline__ void red_or_shared(uint32_t addr, uint32_t v) {
  asm volatile("red.shared.or.b32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}

namespace wide {

constexpr int kWarps = 8;
constexpr int kThreads = 32 * kWarps;

// team of TEAM warps; dynamic shared memory:
// [G][9] matrices | per team: 2 row buffers of BUF bytes | RB x W code words | 2 barriers | 8 partial sums
struct Layout {
  int G, W, RB, BUF, teams;
  int m_off, buf_off, codes_off, bar_off, part_off, bytes;
  __host__ __device__ Layout(int d, int bits, int row_bytes, int team) {
    G = (d + 2) / 3;
    W = (3 * G * bits + 31) / 32;
    teams = kWarps / team;
    BUF = team == 1 ? (row_bytes > 2048 ? row_bytes : 2048) : row_bytes;
    RB = BUF / row_bytes;
    m_off = 0;
    buf_off = ((G * 12 * 4 + 127) / 128) * 128;  // [G][12]: 3x3 matrix padded to 48 bytes
    codes_off = buf_off + teams * 2 * BUF;
    bar_off = codes_off + ((teams * RB * W * 4 + 15) / 16) * 16;
    part_off = bar_off + teams * 2 * 8;
    bytes = part_off + kWarps * 4;
  }
};

// team size: one warp per row (warp-shuffle norm, no CTA barrier per row)
// while every warp's two row buffers fit; the whole CTA beyond that
__host__ __device__ inline int team_of(int d, int bits, int elem_bytes) {
  return Layout(d, bits, d * elem_bytes, 1).bytes <= 227 * 1024 ? 1 : kWarps;
}

template <int TEAM>
__device__ __forceinline__ void team_sync() {
  if (TEAM == 1) __syncwarp();
  else __syncthreads();
}

template <typename TI, typename TO, int BITS, int MODE, int TEAM>
__global__ void __launch_bounds__(kThreads) rq_wide_kernel(RqArgs a) {
  constexpr int K = 1 << BITS;
  constexpr int TT = 32 * TEAM;  // threads per team
  constexpr bool kIn = MODE != RQ_DQ, kOut = MODE != RQ_Q;
  using TB = typename std::conditional<kIn, TI, TO>::type;  // element type held in the row buffers
  __shared__ float s_tau[16], s_mag[16], s_c[16];
  extern __shared__ __align__(128) uint8_t smem[];
  const int d = a.d;
  const Layout L(d, BITS, d * (int)sizeof(TB), TEAM);
  const int G = L.G, W = L.W, RB = L.RB;
  float* s_m = reinterpret_cast<float*>(smem + L.m_off);
  const int warp = threadIdx.x >> 5;
  const int team = warp / TEAM, t = threadIdx.x % TT;
  uint8_t* t_buf = smem + L.buf_off + team * 2 * L.BUF;
  uint32_t* t_codes = reinterpret_cast<uint32_t*>(smem + L.codes_off) + team * RB * W;
  uint64_t* t_bar = reinterpret_cast<uint64_t*>(smem + L.bar_off) + team * 2;
  float* s_part = reinterpret_cast<float*>(smem + L.part_off);

  build_codebook<BITS>(a.centroids, s_tau, s_mag, s_c);
  for (int g = threadIdx.x; g < G; g += kThreads) {
    const float4 r = __ldg(reinterpret_cast<const float4*>(a.rotors) + g);
    rotor_matrix(r.x, r.y, r.z, r.w, s_m + g * 12);
  }
  for (int i = t; i < RB * W; i += TT) t_codes[i] = 0u;
  if (t == 0) {
    mbar_init(&t_bar[0], 1);
    mbar_init(&t_bar[1], 1);
    fence_barrier_init();
  }
  __syncthreads();

  const int64_t n = a.n;
  const int64_t nblk = (n + RB - 1) / RB;
  const int64_t gt = (int64_t)blockIdx.x * L.teams + team, tt = (int64_t)gridDim.x * L.teams;
  const size_t row_bytes = (size_t)d * sizeof(TB);
  const TI* xin = reinterpret_cast<const TI*>(a.x);
  TO* xo = reinterpret_cast<TO*>(a.xhat);
  auto rows_of = [&](int64_t blk) -> int { return (int)(n - blk * RB < RB ? n - blk * RB : RB); };
  auto issue = [&](int64_t blk, int s) {  // thread 0 of the team
    const int rows = rows_of(blk);
    mbar_arrive_expect_tx(&t_bar[s], (uint32_t)(rows * row_bytes));
    if (a.ldx == d) {  // contiguous rows: one copy for the block
      bulk_load(t_buf + s * L.BUF, xin + blk * RB * a.ldx, (uint32_t)(rows * row_bytes), &t_bar[s]);
    } else {
      for (int r = 0; r < rows; ++r)
        bulk_load(t_buf + s * L.BUF + r * row_bytes, xin + (blk * RB + r) * a.ldx, (uint32_t)row_bytes, &t_bar[s]);
    }
  };
  if (kIn && t == 0)
    for (int s = 0; s < 2; ++s)
      if (gt + s * tt < nblk) issue(gt + s * tt, s);

  uint32_t par = 0;
  int it = 0;
  bool failed = false;
  for (int64_t blk = gt; blk < nblk; blk += tt, ++it) {
    const int s = it & 1;
    const int rows = rows_of(blk);
    TB* buf = reinterpret_cast<TB*>(t_buf + s * L.BUF);
    bool ok = true;
    if (kIn) {
      ok = mbar_wait(&t_bar[s], (par >> s) & 1, a.status);
      par ^= 1u << s;
    } else if (t == 0) {
      bulk_wait_read<1>();  // the x_hat store that last used this buffer has read it
    }
    // the team leaves together if a wait ran out
    if (TEAM == 1 ? !__all_sync(0xffffffffu, ok) : !__syncthreads_and(ok)) {
      failed = true;
      break;
    }
    for (int r = 0; r < rows; ++r) {
      const int64_t row = blk * RB + r;
      TB* rb = buf + (size_t)r * d;
      float nrm;
      if constexpr (kIn) {
        float ss = 0.f;
        constexpr int E = 16 / (int)sizeof(TB);
        for (int c = t; c < d / E; c += TT) {
          float f[E];
          Elem<TB>::unpack(reinterpret_cast<const uint4*>(rb)[c], f);
#pragma unroll
          for (int e = 0; e < E; ++e) ss = fmaf(f[e], f[e], ss);
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
        if (TEAM > 1) {
          if ((threadIdx.x & 31) == 0) s_part[warp] = ss;
          __syncthreads();
          ss = 0.f;
#pragma unroll
          for (int w = 0; w < TEAM; ++w) ss += s_part[w];
        }
        nrm = sqrtf(ss);
        if (t == 0 && a.norms_out) a.norms_out[row * a.ldn] = nrm;
      } else {
        nrm = __ldg(a.norms_in + row * a.ldn);
      }
      Quantizer<BITS> q;
      q.scale(s_tau, s_mag, nrm);
      uint32_t* wc = t_codes + r * W;
      const uint32_t wc_a = smem_u32(wc), rb_a = smem_u32(rb), m_a = smem_u32(s_m), c_a = smem_u32(s_c);
      if constexpr (!kIn) {
        // the row's code words, coalesced, into the team's code buffer
        const uint32_t* cin = a.codes_in + row * a.ldc;
        for (int i = t; i < W; i += TT) wc[i] = __ldg(cin + i);
        team_sync<TEAM>();
      }
      // One group: its padded matrix row (three 16-byte loads), its three elements at e_p, its code bits
      // at `bit`; FULL: all three elements are inside the row (every group but a zero-padded last one).
      auto group = [&](auto full, int g, uint32_t m_p, uint32_t e_p, int bit) {
        constexpr bool kFull = decltype(full)::value;
        const uint4 m0 = lds_v4(m_p), m1 = lds_v4(m_p + 16), m2 = lds_v4(m_p + 32);
        const float m[9] = {__uint_as_float(m0.x), __uint_as_float(m0.y), __uint_as_float(m0.z),
                            __uint_as_float(m0.w), __uint_as_float(m1.x), __uint_as_float(m1.y),
                            __uint_as_float(m1.z), __uint_as_float(m1.w), __uint_as_float(m2.x)};
        float c[3];
        if constexpr (kIn) {
          float v[3];
#pragma unroll
          for (int i = 0; i < 3; ++i) v[i] = (kFull || 3 * g + i < d) ? lds_elem<TB>(e_p + i * (int)sizeof(TB)) : 0.f;
          uint32_t bits3 = 0;
#pragma unroll
          for (int i = 0; i < 3; ++i) {
            const float y = fmaf(m[3 * i + 2], v[2], fmaf(m[3 * i + 1], v[1], m[3 * i] * v[0]));
            bits3 |= q(y, c[i]) << (i * BITS);
          }
          red_or_shared(wc_a + (uint32_t)((bit >> 5) * 4), bits3 << (bit & 31));
          if ((bit & 31) + 3 * BITS > 32) red_or_shared(wc_a + (uint32_t)((bit >> 5) * 4 + 4), bits3 >> (32 - (bit & 31)));
        } else {
#pragma unroll
          for (int i = 0; i < 3; ++i) {
            const int b = bit + i * BITS;
            uint32_t v = lds_u32(wc_a + (uint32_t)((b >> 5) * 4)) >> (b & 31);
            if ((b & 31) + BITS > 32) v |= lds_u32(wc_a + (uint32_t)((b >> 5) * 4 + 4)) << (32 - (b & 31));
            c[i] = __uint_as_float(lds_u32(c_a + (v & (K - 1)) * 4)) * nrm;
          }
        }
        if constexpr (kOut) {
#pragma unroll
          for (int i = 0; i < 3; ++i)
            if (kFull || 3 * g + i < d)
              sts_elem<TB>(e_p + i * (int)sizeof(TB), fmaf(m[6 + i], c[2], fmaf(m[3 + i], c[1], m[i] * c[0])));
        }
      };
      // whole groups with addresses advanced by constant strides, then the padded last group
      const int G_full = d / 3;
      int g = t, bit = t * 3 * BITS;
      uint32_t m_p = m_a + (uint32_t)(t * 48), e_p = rb_a + (uint32_t)(3 * t * (int)sizeof(TB));
#pragma unroll 2
      for (; g < G_full; g += TT, bit += TT * 3 * BITS, m_p += TT * 48, e_p += TT * 3 * (int)sizeof(TB))
        group(std::true_type{}, g, m_p, e_p, bit);
      if (g < G) group(std::false_type{}, g, m_p, e_p, bit);
      if constexpr (!kIn) team_sync<TEAM>();  // the code buffer is refilled by the next row
      if constexpr (kIn) {
        team_sync<TEAM>();
        if (a.codes_out)
          for (int i = t; i < W; i += TT) a.codes_out[row * a.ldc + i] = wc[i];
        team_sync<TEAM>();
        for (int i = t; i < W; i += TT) wc[i] = 0u;
      }
    }
    // generic reads (and x_hat writes) of the buffer before the bulk copies that reuse it
    fence_proxy_async_smem();
    team_sync<TEAM>();
    if (t == 0) {
      if constexpr (kOut) {
        if (a.ldo == d) {
          bulk_store(xo + blk * RB * a.ldo, t_buf + s * L.BUF, (uint32_t)(rows * row_bytes));
        } else {
          for (int r = 0; r < rows; ++r)
            bulk_store(xo + (blk * RB + r) * a.ldo, t_buf + s * L.BUF + r * row_bytes, (uint32_t)row_bytes);
        }
        bulk_commit();
      }
      if constexpr (kIn) {
        const int64_t next = blk + 2 * tt;
        if (next < nblk) {
          if (kOut) bulk_wait_read<0>();  // the x_hat store has read the buffer
          issue(next, s);
        }
      }
    }
    team_sync<TEAM>();
  }
  if (t == 0) {
    // after a failed wait, the copy into the other buffer (if any) lands before the team exits
    if (failed && gt + (int64_t)(it + 1) * tt < nblk) mbar_wait(&t_bar[(it + 1) & 1], (par >> ((it + 1) & 1)) & 1, a.status);
    bulk_wait_read<0>();
  }
}

}  // namespace wide

// ============================================================================
// d > 256 with 16-bit rows: a warp per row, each lane a contiguous run of R groups.
// ============================================================================
// Rows stream into shared memory by bulk copy (two buffers per warp). Lane t owns groups
// R t .. R t + R - 1 (R a multiple of 8, so its 3R elements start on a 16-byte boundary and
// d, a multiple of 8, ends on a chunk boundary): it reads its elements as 16-byte chunks,
// rotates group pairs with packed f32x2 FMAs on the pairs' exact sandwich matrices,
// quantizes with the row kernel's binary search (b >= 3) or saturating steps (b <= 2),
// writes x_hat back in place, and ORs its contiguous code bits into the warp's staged code
// words. The pair matrices sit in a per-lane table whose lane stride is padded by 16 bytes,
// so the lanes' 16-byte loads of their own matrices spread over the banks.
namespace run {

constexpr int kWarps = 8;
constexpr int kThreads = 32 * kWarps;

struct Layout {
  int G, W, lane_bytes, row_bytes, buf_off, codes_off, lut_off, bar_off, cb_off, bytes;
  __host__ __device__ Layout(int d, int bits, int R) {
    G = (d + 2) / 3;
    W = (3 * G * bits + 31) / 32;
    lane_bytes = (R / 2) * 80 + 16;
    row_bytes = d * 2;
    buf_off = ((32 * lane_bytes + 127) / 128) * 128;
    codes_off = buf_off + kWarps * 2 * row_bytes;
    lut_off = codes_off + ((kWarps * W * 4 + 15) / 16) * 16;  // dequantize: [warp][16] centroids
    bar_off = lut_off + kWarps * 16 * 4;
    cb_off = bar_off + kWarps * 2 * 8;
    bytes = cb_off + 64 * 4;
  }
};

// run length (groups per lane) for d, 0 when the run kernel does not take d
__host__ __device__ inline int run_groups(int d) {
  if (d <= 256 || d % 8 != 0) return 0;
  const int G = (d + 2) / 3;
  for (int R = 8; R <= 48; R += 8)
    if (32 * R >= G) return R;
  return 0;
}

// two CTAs per SM where their row buffers fit (R <= 24: d <= 2304), so registers are capped at 128
template <typename T, int BITS, int MODE, int R>
__global__ void __launch_bounds__(kThreads, R <= 24 ? 2 : 1) rq_run_kernel(RqArgs a) {
  constexpr int K = 1 << BITS, H = K / 2;
  constexpr bool kIn = MODE != RQ_DQ, kOut = MODE != RQ_Q;
  constexpr bool kScale = !std::is_same<T, __half>::value;  // fp16 norms always lie in [2^-24, 2^20]
  constexpr int E = 8;                 // elements per 16-byte chunk
  constexpr int NE = 3 * R;            // elements (and codes) of a lane's run
  constexpr int NCH = NE / E;          // chunks of the run
  constexpr int NP = R / 2;            // group pairs of the run
  constexpr int CPW = 23 / BITS;       // codes per float window
  constexpr int NWIN = (NE + CPW - 1) / CPW;
  constexpr int WLOC = (NE * BITS + 31) / 32;  // words of the run's own bit stream
  constexpr bool kBisect = BITS >= 3;
  static_assert(R % 8 == 0 && NE % E == 0, "run");

  extern __shared__ __align__(128) uint8_t smem[];
  const int d = a.d;
  const Layout L(d, BITS, R);
  const int G = L.G, W = L.W;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float* s_sc = reinterpret_cast<float*>(smem + L.cb_off);
  float* s_mag = s_sc + 16;
  float* s_cf = s_sc + 32;

  // the per-lane table of pair matrices: lane t, pair p at t * lane_bytes + 80 p, (M_2p, M_2p+1) interleaved
  for (int idx = threadIdx.x; idx < 32 * R; idx += kThreads) {
    const int t = idx / R, gl = idx - t * R, g = R * t + gl;
    float m[9];
    if (g < G) {
      const float4 r4 = __ldg(reinterpret_cast<const float4*>(a.rotors) + g);
      rotor_matrix(r4.x, r4.y, r4.z, r4.w, m);
    } else {
#pragma unroll
      for (int k = 0; k < 9; ++k) m[k] = 0.f;
    }
    float* dst = reinterpret_cast<float*>(smem + t * L.lane_bytes + (gl >> 1) * 80) + (gl & 1);
#pragma unroll
    for (int k = 0; k < 9; ++k) dst[2 * k] = m[k];
    dst[18] = 0.f;
  }
  row::build_consts<BITS>(a.centroids, s_sc, s_mag, s_cf);
  uint8_t* w_buf = smem + L.buf_off + warp * 2 * L.row_bytes;
  uint64_t* w_bar = reinterpret_cast<uint64_t*>(smem + L.bar_off) + warp * 2;
  uint32_t* w_codes = reinterpret_cast<uint32_t*>(smem + L.codes_off) + warp * W;
  float* w_lut = reinterpret_cast<float*>(smem + L.lut_off) + warp * 16;
  for (int i = lane; i < W; i += 32) w_codes[i] = 0u;
  if (lane == 0) {
    mbar_init(&w_bar[0], 1);
    mbar_init(&w_bar[1], 1);
    fence_barrier_init();
  }
  __syncthreads();

  const int64_t n = a.n;
  const int64_t gw = (int64_t)blockIdx.x * kWarps + warp, tw = (int64_t)gridDim.x * kWarps;
  const T* xin = reinterpret_cast<const T*>(a.x);
  T* xo_g = reinterpret_cast<T*>(a.xhat);
  const uint32_t rb_bytes = (uint32_t)L.row_bytes;
  auto issue = [&](int64_t row, int s) {  // lane 0
    mbar_arrive_expect_tx(&w_bar[s], rb_bytes);
    bulk_load(w_buf + s * L.row_bytes, xin + row * a.ldx, rb_bytes, &w_bar[s]);
  };
  if (kIn && lane == 0)
    for (int s = 0; s < 2; ++s)
      if (gw + s * tw < n) issue(gw + s * tw, s);

  const int e0 = NE * lane;  // the run's first element
  const uint32_t tab_a = smem_u32(smem) + (uint32_t)(lane * L.lane_bytes);
  const uint32_t codes_a = smem_u32(w_codes);
  const int base = NE * BITS * lane;  // the run's first code bit in the row's stream
  float sc[H > 1 ? H - 1 : 1];
#pragma unroll
  for (int j = 0; j < H - 1; ++j) sc[j] = s_sc[j];
  uint32_t par = 0;
  int it = 0;
  bool failed = false;
  for (int64_t row = gw; row < n; row += tw, ++it) {
    const int s = it & 1;
    uint8_t* rb = w_buf + s * L.row_bytes;
    const uint32_t run_a = smem_u32(rb) + (uint32_t)(e0 * 2);
    bool ok = true;
    if constexpr (kIn) {
      ok = mbar_wait(&w_bar[s], (par >> s) & 1, a.status);
      par ^= 1u << s;
    } else if (lane == 0) {
      bulk_wait_read<1>();  // the x_hat store that last used this buffer has read it
    }
    if (!__all_sync(0xffffffffu, ok)) {
      failed = true;
      break;
    }
    auto chunk_in = [&](int c) { return e0 + E * c < d; };  // d and e0 are multiples of 8

    // ---------------------------------------------------------------- per-row scale
    float xs = 1.f, nrm, nq;
    if constexpr (kIn) {
      float2 acc[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
      for (int c = 0; c < NCH; ++c) {
        if (chunk_in(c)) {
          if constexpr (std::is_same<T, __half>::value) {  // fp16 squares straight into the fp32 sums
            const uint4 c4 = lds_v4(run_a + 16u * c);
            const uint32_t cw[4] = {c4.x, c4.y, c4.z, c4.w};
#pragma unroll
            for (int k = 0; k < 4; ++k) sq_acc_f16x2(cw[k], acc[k & 1].x, acc[k & 1].y);
          } else {
            float f[E];
            Elem<T>::unpack(lds_v4(run_a + 16u * c), f);
#pragma unroll
            for (int k = 0; k < E / 2; ++k) {
              const float2 v = make_float2(f[2 * k], f[2 * k + 1]);
              acc[k & 1] = __ffma2_rn(v, v, acc[k & 1]);
            }
          }
        }
      }
      float ss = (acc[0].x + acc[1].x) + (acc[0].y + acc[1].y);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
      if (kScale && !(ss >= 0x1p-100f && ss <= 0x1p100f)) {
        xs = ss < 1.f ? 0x1p100f : 0x1p-100f;
        ss = 0.f;
#pragma unroll 1
        for (int c = 0; c < NCH; ++c) {
          if (chunk_in(c)) {
            float f[E];
            Elem<T>::unpack(lds_v4(run_a + 16u * c), f);
            for (int k = 0; k < E; ++k) ss = fmaf(f[k] * xs, f[k] * xs, ss);
          }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
      }
      nq = sqrtf(ss);
      nrm = kScale ? nq / xs : nq;
    } else {
      nrm = __ldg(a.norms_in + row * a.ldn);
      nq = nrm;
      const uint32_t* cin = a.codes_in + row * a.ldc;
      for (int i = lane; i < W; i += 32) w_codes[i] = __ldg(cin + i);
    }

    // scaled magnitudes (the row kernel's sequence, so that quantize and dequantize agree bit for bit)
    const float mn0 = __fmul_rn(s_mag[0], nrm);
    float dl[H > 1 ? H - 1 : 1];
    Bisect<kBisect ? BITS : 3> bs;
    if constexpr (kBisect) {
      float Mj[H];
#pragma unroll
      for (int j = 0; j < H; ++j) Mj[j] = __fmul_rn(s_mag[j], nrm);
      bs.magnitudes(Mj);
      bs.thresholds(sc);
    } else {
      float prev = mn0;
#pragma unroll
      for (int j = 1; j < H; ++j) {
        const float cur = __fmul_rn(s_mag[j], nrm);
        dl[j - 1] = __fsub_rn(cur, prev);
        prev = cur;
      }
    }
    uint32_t lw[WLOC + 1];  // dequantize: the run's code words, aligned to its first code
    if constexpr (!kIn) {
      if (lane < H) {
        float ch;
        if constexpr (kBisect) {
          ch = bs.mag(lane);
        } else {
          ch = mn0;
#pragma unroll
          for (int j = 0; j < H - 1; ++j)
            if (j < lane) ch = __fadd_rn(ch, dl[j]);
        }
        w_lut[H + lane] = ch;
        w_lut[H - 1 - lane] = -ch;
      }
      __syncwarp();
      const int w0 = base >> 5, sh = base & 31;
      uint32_t raw[WLOC + 1];
#pragma unroll
      for (int j = 0; j <= WLOC; ++j) raw[j] = (w0 + j < W) ? lds_u32(codes_a + 4u * (uint32_t)(w0 + j)) : 0u;
#pragma unroll
      for (int j = 0; j <= WLOC; ++j)
        lw[j] = sh == 0 ? raw[j] : ((raw[j] >> sh) | (j < WLOC ? raw[j + 1] << (32 - sh) : 0u));
    }
    const uint32_t lut_a = smem_u32(w_lut);
    const float srow = nq > 0.f ? __fdiv_rn(row::kB, nq) : 0.f;
    const float shv = -fmaf(row::kShift, nq, 0x1p-126f);
    const float2 shift2 = make_float2(shv, shv);
    float win[NWIN];
#pragma unroll
    for (int w = 0; w < NWIN; ++w) win[w] = row::kWindow0;

    // ---------------------------------------------------------------- group pairs of the run
    float xe[NE + 6], xo[NE];
#pragma unroll
    for (int p = 0; p < NP; ++p) {
      if constexpr (kIn) {
#pragma unroll
        for (int e = 6 * p; e < 6 * p + 6; ++e)
          if (e % E == 0) {
            if (chunk_in(e / E)) {
              Elem<T>::unpack(lds_v4(run_a + 16u * (uint32_t)(e / E)), &xe[e]);
              if constexpr (kScale) {
#pragma unroll
                for (int k = 0; k < E; ++k) xe[e + k] *= xs;
              }
            } else {
#pragma unroll
              for (int k = 0; k < E; ++k) xe[e + k] = 0.f;
            }
          }
      }
      float2 M[10];
#pragma unroll
      for (int q = 0; q < 5; ++q) {
        const uint4 t4 = lds_v4(tab_a + (uint32_t)((p * 5 + q) * 16));
        M[2 * q] = make_float2(__uint_as_float(t4.x), __uint_as_float(t4.y));
        M[2 * q + 1] = make_float2(__uint_as_float(t4.z), __uint_as_float(t4.w));
      }
      // groups R lane + 2p (lane x) and R lane + 2p + 1 (lane y); beyond G neither codes nor elements
      const bool gx = R * lane + 2 * p < G, gy = R * lane + 2 * p + 1 < G;
      float2 C[3];
      if constexpr (kIn) {
        float2 V[3];
#pragma unroll
        for (int j = 0; j < 3; ++j) V[j] = make_float2(xe[6 * p + j], xe[6 * p + 3 + j]);
#pragma unroll
        for (int i = 0; i < 3; ++i) {
          const float2 Y =
              __ffma2_rn(M[3 * i + 2], V[2], __ffma2_rn(M[3 * i + 1], V[1], __ffma2_rn(M[3 * i], V[0], shift2)));
          float2 m2 = make_float2(mn0, mn0);
          float2 cnt = make_float2(0.5f, 0.5f);
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
          C[i] = __fmul2_rn(m2, sg);
          const float2 code = __ffma2_rn(sg, cnt, make_float2(H - 0.5f, H - 0.5f));
          const int kx = 6 * p + i, ky = 6 * p + 3 + i;  // code indices in the run
          if (gx) win[kx / CPW] = fmaf(code.x, (float)(1u << (BITS * (kx % CPW))), win[kx / CPW]);
          if (gy) win[ky / CPW] = fmaf(code.y, (float)(1u << (BITS * (ky % CPW))), win[ky / CPW]);
        }
      } else {
#pragma unroll
        for (int i = 0; i < 3; ++i) {
          const int kx = 6 * p + i, ky = 6 * p + 3 + i;
          const float cx = gx ? __uint_as_float(lds_u32(lut_a + 4u * get_code<BITS, WLOC + 1>(lw, kx))) : 0.f;
          const float cy = gy ? __uint_as_float(lds_u32(lut_a + 4u * get_code<BITS, WLOC + 1>(lw, ky))) : 0.f;
          C[i] = make_float2(cx, cy);
        }
      }
      if constexpr (kOut) {
#pragma unroll
        for (int i = 0; i < 3; ++i) {
          const float2 X = __ffma2_rn(M[6 + i], C[2], __ffma2_rn(M[3 + i], C[1], __fmul2_rn(M[i], C[0])));
          xo[6 * p + i] = X.x;
          xo[6 * p + 3 + i] = X.y;
        }
#pragma unroll
        for (int e = 6 * p; e < 6 * p + 6; ++e)
          if (e % E == E - 1 && chunk_in(e / E)) sts_v4(run_a + 16u * (uint32_t)(e / E), Elem<T>::pack(&xo[e - (E - 1)]));
      }
    }

    // ---------------------------------------------------------------- outputs
    if constexpr (kIn) {
      // the run's bit stream (codes past the row's 3G left at zero), shifted to its place in the row's words
      uint32_t wl[WLOC];
#pragma unroll
      for (int w = 0; w < WLOC; ++w) wl[w] = 0u;
#pragma unroll
      for (int w = 0; w < NWIN; ++w) {
        const uint32_t v = __float_as_uint(win[w]) & 0x7fffffu;
        const int bo = w * CPW * BITS;
        wl[bo >> 5] |= v << (bo & 31);
        if ((bo & 31) + CPW * BITS > 32 && (bo >> 5) + 1 < WLOC) wl[(bo >> 5) + 1] |= v >> (32 - (bo & 31));
      }
      const int w0 = base >> 5, sh = base & 31;
#pragma unroll
      for (int j = 0; j <= WLOC; ++j) {
        const uint32_t lo = j < WLOC ? wl[j] << sh : 0u;
        const uint32_t hi = (j > 0 && sh != 0) ? wl[j - 1] >> (32 - sh) : 0u;
        const uint32_t v = lo | hi;
        if (v != 0u && w0 + j < W) red_or_shared(codes_a + 4u * (uint32_t)(w0 + j), v);
      }
      if (lane == 0 && a.norms_out) a.norms_out[row * a.ldn] = nrm;
    }
    fence_proxy_async_smem();
    __syncwarp();
    if constexpr (kIn) {
      if (a.codes_out) {
        uint32_t* cout = a.codes_out + row * a.ldc;
        for (int i = lane; i < W; i += 32) cout[i] = w_codes[i];
      }
      __syncwarp();
      for (int i = lane; i < W; i += 32) w_codes[i] = 0u;
    }
    if (lane == 0) {
      if constexpr (kOut) {
        bulk_store(xo_g + row * a.ldo, rb, rb_bytes);
        bulk_commit();
      }
      if constexpr (kIn) {
        const int64_t next = row + 2 * tw;
        if (next < n) {
          if (kOut) bulk_wait_read<0>();  // the x_hat store has read the buffer
          issue(next, s);
        }
      }
    }
    __syncwarp();
  }
  if (lane == 0) {
    // after a failed wait, the copy into the other buffer (if any) lands before the warp exits
    if (failed && gw + (int64_t)(it + 1) * tw < n) mbar_wait(&w_bar[(it + 1) & 1], (par >> ((it + 1) & 1)) & 1, a.status);
    bulk_wait_all<0>();
  }
}

}  // namespace run

// ============================================================================
// Launch helpers (host)
// ============================================================================
template <typename T, int BITS, int MODE, bool RING, int DD, int L>
static cudaError_t launch_row_s(const CUtensorMap& mx, const CUtensorMap& mo, const RqArgs& a, cudaStream_t st,
                                int num_sms) {
  using SM = row::Smem<T, BITS, MODE, RING, DD, L>;
  using SH = row::Shape<T, BITS, MODE, RING>;
  auto kern = rq_row_kernel<T, BITS, MODE, RING, DD, L>;
  static int blocks_per_sm = -1;
  if (blocks_per_sm < 0) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SM::alloc);
    if (e != cudaSuccess) return e;
    int b = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, kern, SH::kRows, SM::alloc);
    if (e != cudaSuccess) return e;
    blocks_per_sm = b < 1 ? 1 : b;
  }
  const int64_t nsub = (a.n + row::kWR - 1) / row::kWR;
  // ring: every CTA starts with at least one sub-tile (its warp 0 takes sub-tile blockIdx.x)
  const int64_t want = SH::kRing ? nsub : (nsub + SH::kWarps - 1) / SH::kWarps;
  const int64_t grid = std::min<int64_t>(want, (int64_t)num_sms * blocks_per_sm);
  return launch_pdl(kern, (unsigned)grid, SH::kRows, SM::alloc, st, mx, mo, a);
}

int rq_row_box_rows() { return row::kWR; }

bool rq_row_dims(int d, kvrq_dtype dt) { return d == 128 || (d == 256 && dt != KVRQ_F32); }

// The ring shape exists for d = 128, 16-bit rows, quantize or fused, and buffers that fit.
template <typename T, int BITS, int MODE, int DD, int L>
constexpr bool can_ring() {
  if constexpr (DD == 128 && MODE != RQ_DQ && sizeof(T) == 2)
    return row::Smem<T, BITS, MODE, true, DD, L>::fits;
  else
    return false;
}

template <typename T, int BITS, int MODE, int DD, int L>
static cudaError_t launch_row(const CUtensorMap& mx, const CUtensorMap& mo, const RqArgs& a, cudaStream_t st,
                              int num_sms) {
  // the ring pays off once every warp of the GPU has two sub-tiles or more
  if constexpr (can_ring<T, BITS, MODE, DD, L>()) {
    if ((a.n + row::kWR - 1) / row::kWR >= 2 * row::Shape<T, BITS, MODE, true>::kWarps * (int64_t)num_sms)
      return launch_row_s<T, BITS, MODE, true, DD, L>(mx, mo, a, st, num_sms);
  }
  return launch_row_s<T, BITS, MODE, false, DD, L>(mx, mo, a, st, num_sms);
}

template <typename TI, typename TO, int BITS, int MODE, int TEAM>
static cudaError_t launch_wide_t(const RqArgs& a, cudaStream_t st, int num_sms) {
  using TB = typename std::conditional<MODE != RQ_DQ, TI, TO>::type;
  const wide::Layout L(a.d, BITS, a.d * (int)sizeof(TB), TEAM);
  auto kern = wide::rq_wide_kernel<TI, TO, BITS, MODE, TEAM>;
  static int set_bytes = 0;
  if (L.bytes > set_bytes) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L.bytes);
    if (e != cudaSuccess) return e;
    set_bytes = L.bytes;
  }
  int per_sm = 0;
  cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, wide::kThreads, L.bytes);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) per_sm = 1;
  const int64_t nblk = (a.n + L.RB - 1) / L.RB;
  const int64_t grid = std::min<int64_t>((nblk + L.teams - 1) / L.teams, (int64_t)num_sms * per_sm);
  kern<<<(unsigned)grid, wide::kThreads, L.bytes, st>>>(a);
  return cudaGetLastError();
}

template <typename TI, typename TO, int BITS, int MODE>
static cudaError_t launch_wide(const RqArgs& a, cudaStream_t st, int num_sms) {
  using TB = typename std::conditional<MODE != RQ_DQ, TI, TO>::type;
  if (wide::team_of(a.d, BITS, (int)sizeof(TB)) == 1) return launch_wide_t<TI, TO, BITS, MODE, 1>(a, st, num_sms);
  return launch_wide_t<TI, TO, BITS, MODE, wide::kWarps>(a, st, num_sms);
}

// Shared memory the bulk-copy kernel needs for d (0 when it cannot take d).
int rq_wide_smem_bytes(int d, int bits, int elem_bytes) {
  if ((d * elem_bytes) % 16 != 0 || d * elem_bytes > 16384) return 0;
  const wide::Layout L(d, bits, d * elem_bytes, wide::team_of(d, bits, elem_bytes));
  return L.bytes <= 227 * 1024 ? L.bytes : 0;
}

template <typename TI, typename TO, int BITS, int MODE>
static cudaError_t launch_general(const RqArgs& a, cudaStream_t st, int num_sms) {
  const int64_t warps = a.n;
  const int64_t blocks = std::min<int64_t>((warps + 7) / 8, (int64_t)num_sms * 8);
  rq_general_kernel<TI, TO, BITS, MODE><<<(unsigned)blocks, 256, 0, st>>>(a);
  return cudaGetLastError();
}

template <typename T, int MODE, int DD, int L = 3>
static cudaError_t row_by_bits(int bits, const CUtensorMap& mx, const CUtensorMap& mo, const RqArgs& a,
                               cudaStream_t st, int sms) {
  switch (bits) {
    case 1: return launch_row<T, 1, MODE, DD, L>(mx, mo, a, st, sms);
    case 2: return launch_row<T, 2, MODE, DD, L>(mx, mo, a, st, sms);
    case 3: return launch_row<T, 3, MODE, DD, L>(mx, mo, a, st, sms);
    default: return launch_row<T, 4, MODE, DD, L>(mx, mo, a, st, sms);
  }
}

template <int MODE>
static cudaError_t row_by_type(kvrq_dtype dt, int bits, const CUtensorMap& mx, const CUtensorMap& mo,
                               const RqArgs& a, cudaStream_t st, int sms) {
  if (a.d == 256) {  // 16-bit rows only (rq_row_dims)
    if (dt == KVRQ_F16) return row_by_bits<__half, MODE, 256>(bits, mx, mo, a, st, sms);
    return row_by_bits<__nv_bfloat16, MODE, 256>(bits, mx, mo, a, st, sms);
  }
  if (a.codes_per_group == 4) {  // the four-grade layout (d = 128 only, checked on the host)
    switch (dt) {
      case KVRQ_F32: return row_by_bits<float, MODE, 128, 4>(bits, mx, mo, a, st, sms);
      case KVRQ_F16: return row_by_bits<__half, MODE, 128, 4>(bits, mx, mo, a, st, sms);
      default: return row_by_bits<__nv_bfloat16, MODE, 128, 4>(bits, mx, mo, a, st, sms);
    }
  }
  switch (dt) {
    case KVRQ_F32: return row_by_bits<float, MODE, 128>(bits, mx, mo, a, st, sms);
    case KVRQ_F16: return row_by_bits<__half, MODE, 128>(bits, mx, mo, a, st, sms);
    default: return row_by_bits<__nv_bfloat16, MODE, 128>(bits, mx, mo, a, st, sms);
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

template <typename T, int BITS, int MODE, int R>
static cudaError_t launch_run_t(const RqArgs& a, cudaStream_t st, int num_sms) {
  const run::Layout L(a.d, BITS, R);
  auto kern = run::rq_run_kernel<T, BITS, MODE, R>;
  static int set_bytes = 0;
  if (L.bytes > set_bytes) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L.bytes);
    if (e != cudaSuccess) return e;
    set_bytes = L.bytes;
  }
  int per_sm = 0;
  cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, run::kThreads, L.bytes);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) per_sm = 1;
  const int64_t grid = std::min<int64_t>((a.n + run::kWarps - 1) / run::kWarps, (int64_t)num_sms * per_sm);
  kern<<<(unsigned)grid, run::kThreads, L.bytes, st>>>(a);
  return cudaGetLastError();
}

// Run length of the run kernel for 16-bit rows of d, or 0 (the bulk-copy kernel takes d).
static int run_length(int d, int bits) {
  int R = run::run_groups(d);
  if (R == 32 || R == 40) R = 48;  // instantiated lengths: 8, 16, 24, 48
  if (R == 0 || run::Layout(d, bits, R).bytes > 227 * 1024) return 0;
  return R;
}

template <typename T, int BITS, int MODE>
static cudaError_t launch_run(int R, const RqArgs& a, cudaStream_t st, int sms) {
  switch (R) {
    case 8: return launch_run_t<T, BITS, MODE, 8>(a, st, sms);
    case 16: return launch_run_t<T, BITS, MODE, 16>(a, st, sms);
    case 24: return launch_run_t<T, BITS, MODE, 24>(a, st, sms);
    default: return launch_run_t<T, BITS, MODE, 48>(a, st, sms);
  }
}

template <typename TI, typename TO, int MODE>
static cudaError_t gen_by_bits(int bits, const RqArgs& a, cudaStream_t st, int sms) {
  using TB = typename std::conditional<MODE != RQ_DQ, TI, TO>::type;
  if constexpr (sizeof(TB) == 2) {
    // 16-bit rows of d > 256: a warp per row, a contiguous run of groups per lane
    const int R = a.wide ? run_length(a.d, bits) : 0;
    if (R > 0) {
      switch (bits) {
        case 1: return launch_run<TB, 1, MODE>(R, a, st, sms);
        case 2: return launch_run<TB, 2, MODE>(R, a, st, sms);
        case 3: return launch_run<TB, 3, MODE>(R, a, st, sms);
        default: return launch_run<TB, 4, MODE>(R, a, st, sms);
      }
    }
  }
  if (a.wide) {
    switch (bits) {
      case 1: return launch_wide<TI, TO, 1, MODE>(a, st, sms);
      case 2: return launch_wide<TI, TO, 2, MODE>(a, st, sms);
      case 3: return launch_wide<TI, TO, 3, MODE>(a, st, sms);
      default: return launch_wide<TI, TO, 4, MODE>(a, st, sms);
    }
  }
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
