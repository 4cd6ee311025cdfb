// Fused decode attention from a packed KV cache on tcgen05 tensor cores.
//   out_(h,g) = sum_t softmax_t(scale * <q_(h,g), k_hat_t>) * v_hat_t
// ["TurboQuant и PolarQuant", "Проблема KV-кэша в трансформерах": softmax(Q K^T / sqrt(d)) V;
//  "TurboQuant + RotorQuant", "When to Use Which": attention computed from the compressed
//  indices; "How TurboQuant Works": <q, k> ~ <q, k_mse> + ||r|| sqrt(pi/2)/m <S q, sign(S r)>]
//
// Both contractions of a 128-token tile run on the tensor cores; nothing is dequantized
// into global memory:
//   MMA1  S[128 tokens x 16] = A1 . B1^T, K = 128 (+128 for the QJL signs, +16 padding
//         for RotorQuant keys): A1 = the tile's decoded keys (fp16 centroids and +-1
//         signs) written by the decoding threads straight into tensor memory, one token
//         per lane; B1 = the head's rotated queries q' (and T q') in shared memory.
//   MMA2  O[128 coordinates x 16] += A2 . B2^T, K = 128 tokens: A2 = the tile's decoded
//         RotorQuant values in the rotated domain (fp16 centroids, MN-major in shared
//         memory: token t is K row t); B2 = the softmax weights w_t ||v_t|| (fp16).
// The softmax is online: per tile the warpgroup forms its running maximum, rescales
// the value accumulator in tensor memory when the maximum grows, and keeps the weight
// sums per thread (reduced once per chunk). The 129th rotated value coordinate (the
// rotor pad) is summed on the CUDA cores. Each warpgroup leaves one partial (max,
// weight sum, rotated value sums) per work item for the merge kernel, which applies
// the inverse sandwich once per query row.
//
// B200 shape: a persistent CTA of three decode warpgroups per SM (tensor memory holds
// A1 and both accumulators of each; 168 registers per thread). Each warpgroup is a
// worker of its own: it takes (KV head, token range) work items in turn, writes the
// head's query operand B1 into its own buffer, streams the item's code rows, sign rows
// and norms by bulk copy into its own stage (the next tile's copy lands while the
// current tile is computed; an item's first copy while B1 is written), and leaves one
// partial per item. Its first thread issues the copies and both MMAs. Every wait is
// bounded; a time-out is recorded in the device status word and the warpgroup drains
// its copies and MMAs and stops.

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "attn_launch.h"
#include "kvrq_device.cuh"
#include "score_launch.h"
#include "tc_decode.cuh"

namespace kvrq {
namespace attn_tc {

constexpr int kRows = 128;         // tokens per tile = TMEM lanes
constexpr int kNWG = kAttnTcParts;  // decode warpgroups per CTA (one partial each per work item)
constexpr int kThreads = 128 * kNWG;
constexpr int kStages = 1;          // copy stages per warpgroup (a refill lands while the tile is computed)
constexpr int NB = 16;      // MMA N: query rows (and, for prod, their T q' rows)
constexpr int kNcv = 129;   // stored RotorQuant value coordinates (3G at d = 128)
constexpr uint32_t kTmemCols = 512;

// A decode table with `RDIV` times fewer replicas than Dec (lanes l and l + R share one, a 2-way bank
// conflict for RDIV = 2): line = the R replicas of one entry.
template <int BITS, int RDIV>
struct Lut {
  using D = Dec<BITS>;
  static constexpr int R = D::R / RDIV;
  static constexpr int LINE = R * D::EB;     // bytes per entry
  static constexpr int LSH = LINE == 128 ? 7 : (LINE == 64 ? 6 : 5);
  static_assert((1 << LSH) == LINE, "line");
  static constexpr int BYTES = D::ENT * LINE;
};

template <int KM, int KB, int VB>
struct Cfg {
  using KL = Lut<KB, 2>;
  using VL = Lut<VB, 1>;
  static constexpr bool kProd = KM == KVRQ_TQ_PROD;
  static constexpr int GMAX = kProd ? NB / 2 : NB;  // query rows per KV head
  static constexpr int NCODE = KM == KVRQ_RQ_MSE ? 129 : 128;
  static constexpr int KC = KM == KVRQ_RQ_MSE ? 144 : 128;  // MMA1 K of the centroid part
  static constexpr int K = KC + (kProd ? 128 : 0);
  static constexpr int KAP = (K / 2 + 31) / 32 * 32;        // A1 columns (fp16 pairs), 32-aligned
  static constexpr int KBOX = (K + 63) / 64;
  static constexpr int WK = (NCODE * KB + 31) / 32;  // key code words
  static constexpr int NS = kProd ? 4 : 0;           // sign words (m = 128)
  static constexpr int WV = (kNcv * VB + 31) / 32;   // value code words
  static constexpr int B_BOX = NB * 128;             // 64 K elements x NB rows
  static constexpr int WCOLS = KAP + 2 * NB;         // A1, S, O
  static_assert(kNWG * WCOLS <= (int)kTmemCols, "tensor memory");
  // a stage: key codes [128][WK], signs [128][NS], value codes [128][WV], key norms, gammas, value norms
  static constexpr int st_s = kRows * WK;
  static constexpr int st_v = st_s + kRows * NS;
  static constexpr int st_kn = st_v + kRows * WV;
  static constexpr int st_kg = st_kn + kRows;
  static constexpr int st_vn = st_kg + kRows;
  static constexpr int stage_words = st_vn + kRows;
  // shared memory (from a 1024-aligned base)
  static constexpr int klut_off = 0;
  static constexpr int slut_off = klut_off + KL::BYTES;
  static constexpr int SLINE = 64;  // signs: byte -> 8 x (+1/-1) (16 bytes), 4 replicas
  static constexpr int vlut_off = slut_off + (kProd ? 256 * SLINE : 0);
  static constexpr int vc_off = vlut_off + VL::BYTES;  // fp32 value centroids [16]
  static constexpr int b1_off = ((vc_off + 64 + 1023) / 1024) * 1024;
  static constexpr int B1_BYTES = ((KBOX * B_BOX + 1023) / 1024) * 1024;       // per wg
  static constexpr int A2_ATOM = kRows * 128;  // 64 coordinates x 128 tokens
  static constexpr int a2_off = b1_off + kNWG * B1_BYTES;                         // [wg][2 atoms]
  static constexpr int B2_BYTES = 2 * B_BOX;                                     // 128 tokens x NB rows
  static constexpr int b2_off = a2_off + kNWG * 2 * A2_ATOM;                      // [wg]
  static constexpr int stage_off = b2_off + kNWG * B2_BYTES;                      // [wg][stage]
  static constexpr int red_off = stage_off + kNWG * kStages * stage_words * 4;    // [wg][warp][GMAX]
  static constexpr int bar_off = red_off + kNWG * 4 * GMAX * 4;
  static constexpr int nbars = kNWG * (kStages + 2);  // per wg: stages, MMA1 done, MMA2 done
  static constexpr int tmem_off = bar_off + nbars * 8;
  static constexpr int alloc = tmem_off + 16 + 1024;
  static constexpr bool fits = alloc <= 227 * 1024;
};

template <int KM, int KB, int VB>
__global__ void __launch_bounds__(kThreads, 1) attn_tc_kernel(AttnArgs a) {
  using C = Cfg<KM, KB, VB>;
  static_assert(C::fits, "shared memory");
  using DK = Dec<KB>;
  using DV = Dec<VB>;
  using KL = typename C::KL;
  using VL = typename C::VL;
  constexpr int WK = C::WK, NS = C::NS, WV = C::WV, GMAX = C::GMAX, K = C::K, KC = C::KC;
  constexpr bool kProd = C::kProd;
  constexpr uint32_t kId1 = umma_idesc_f16(false, false, false, NB, kRows);
  constexpr uint32_t kId2 = umma_idesc_f16(false, false, false, NB, kRows) | (1u << 15);  // A MN-major

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* s_bar = reinterpret_cast<uint64_t*>(smem + C::bar_off);
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + C::tmem_off);
  float* s_vc = reinterpret_cast<float*>(smem + C::vc_off);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int w = warp >> 2, q4 = warp & 3, r = tid & 127;
  const int group = a.group;

  if (tid == 0) {
    for (int i = 0; i < C::nbars; ++i) mbar_init(&s_bar[i], 1);
    fence_barrier_init();
  }
  if (warp == 0) tmem_alloc(s_tmem, kTmemCols);
  // decode tables, replicated per lane group (see Dec)
  for (int i = tid; i < KL::BYTES / 2; i += kThreads) {  // half j of an entry line: code j % P of the field
    const int e = i / (KL::LINE / 2), j = (i % (KL::LINE / 2)) % DK::P;
    reinterpret_cast<__half*>(smem + C::klut_off)[i] = __float2half_rn(a.k_centroids[(e >> (j * KB)) & ((1 << KB) - 1)]);
  }
  if (kProd)
    for (int i = tid; i < 256 * C::SLINE / 2; i += kThreads) {
      const int e = i / (C::SLINE / 2), j = (i % (C::SLINE / 2)) % 8;
      reinterpret_cast<__half*>(smem + C::slut_off)[i] = __float2half_rn(((e >> j) & 1) ? 1.f : -1.f);
    }
  for (int i = tid; i < VL::BYTES / 2; i += kThreads) {
    const int e = i / (VL::LINE / 2), j = (i % (VL::LINE / 2)) % DV::P;
    reinterpret_cast<__half*>(smem + C::vlut_off)[i] = __float2half_rn(a.v_centroids[(e >> (j * VB)) & ((1 << VB) - 1)]);
  }
  if (tid < (1 << VB)) s_vc[tid] = a.v_centroids[tid];
  // B2 rows >= GMAX (the QJL rows of the logit operand have no weights) stay zero for the whole kernel
  if constexpr (GMAX < NB)
    for (int i = tid; i < kNWG * 2 * (NB - GMAX) * 32; i += kThreads) {
      const int wg = i / (2 * (NB - GMAX) * 32), rem = i - wg * 2 * (NB - GMAX) * 32;
      const int box = rem / ((NB - GMAX) * 32), rr = rem - box * (NB - GMAX) * 32;
      reinterpret_cast<uint32_t*>(smem + C::b2_off + wg * C::B2_BYTES + box * C::B_BOX + GMAX * 128)[rr] = 0u;
    }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;

  // this warpgroup's tensor memory, buffers and barriers
  uint64_t* bar_st = s_bar + w * (kStages + 2);
  uint64_t* bar1 = bar_st + kStages;
  uint64_t* bar2 = bar1 + 1;
  const uint32_t a1_mma = tmem + (uint32_t)(w * C::WCOLS);
  const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
  const uint32_t a1_t = a1_mma + lane_off;
  const uint32_t s_t = a1_t + (uint32_t)C::KAP;
  const uint32_t o_t = s_t + (uint32_t)NB;
  const uint32_t s_mma = a1_mma + (uint32_t)C::KAP;
  const uint32_t o_mma = s_mma + (uint32_t)NB;
  const uint32_t b1_s = smem_u32(smem + C::b1_off + w * C::B1_BYTES);
  const uint32_t a2_s = smem_u32(smem + C::a2_off + w * 2 * C::A2_ATOM);
  const uint32_t b2_s = smem_u32(smem + C::b2_off + w * C::B2_BYTES);
  uint32_t* w_stage = reinterpret_cast<uint32_t*>(smem + C::stage_off) + w * kStages * C::stage_words;
  const uint32_t klut_l = smem_u32(smem + C::klut_off) + (uint32_t)((lane % KL::R) * DK::EB);
  const uint32_t slut_l = smem_u32(smem + C::slut_off) + (uint32_t)((lane & 3) * 16);
  const uint32_t vlut_l = smem_u32(smem + C::vlut_off) + (uint32_t)((lane % VL::R) * DV::EB);
  float* red = reinterpret_cast<float*>(smem + C::red_off) + w * 4 * GMAX;

  const int64_t items_per_head = (a.n_tokens + a.tokens_per_cta - 1) / a.tokens_per_cta;
  const int64_t n_items = a.n_heads * items_per_head;
  const uint32_t lim = a.spin_limit < 0 ? kSpinLimit : (uint32_t)a.spin_limit;  // tile-copy waits (the drain: default)
  uint32_t par_st = 0;  // bit s: parity of stage s's next completion
  uint32_t n1 = 0, n2 = 0;  // MMA1 / MMA2 completions waited for so far
  int slot = 0;             // stage of this warpgroup's next tile
  bool ok = true;

  // each warpgroup is a worker of its own: items w * gridDim.x + blockIdx.x, then every
  // kNWG * gridDim.x-th one
  const int64_t n_workers = (int64_t)kNWG * gridDim.x;
  for (int64_t item = (int64_t)w * gridDim.x + blockIdx.x; item < n_items; item += n_workers) {
    const int64_t head = item / items_per_head;
    const int64_t chunk = item - head * items_per_head;
    const int64_t row0 = head * group;
    const int64_t t_begin = chunk * a.tokens_per_cta;
    const PagedHead ph = paged_head(head, a.n_tokens, a.block_tables, a.ld_table, a.seq_lens, a.page_tokens,
                                    a.n_seqs, a.kv_heads);
    const int64_t t_end = ph.n_tokens < t_begin + a.tokens_per_cta ? ph.n_tokens : t_begin + a.tokens_per_cta;
    const int ntiles = t_end > t_begin ? (int)((t_end - t_begin + kRows - 1) / kRows) : 0;
    const uint32_t* kbase = a.k_codes + ph.pool_head * a.k_head_stride;
    const uint32_t* sbase = kProd ? a.k_signs + ph.pool_head * a.s_head_stride : nullptr;
    const uint32_t* vbase = a.v_codes + ph.pool_head * a.v_head_stride;
    const float* knb = a.k_norms + ph.pool_head * a.tok_head_stride;
    const float* kgb = kProd ? a.k_gammas + ph.pool_head * a.tok_head_stride : nullptr;
    const float* vnb = a.v_norms + ph.pool_head * a.tok_head_stride;
    // a paged tile is copied one page segment (min(page, 128) rows) at a time: pages of a power of two >= 16
    // slots start 16-byte aligned and split a 128-token tile evenly
    const int seg = !ph.table ? kRows : (ph.ptok < kRows ? ph.ptok : kRows);
    auto al16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; };
    // a full tile's rows are contiguous, 16-byte aligned blocks when the rows are unpadded
    const bool bulk = (!ph.table || ph.shift >= 4) && a.ldk == WK && (!kProd || a.lds == NS) && a.ldv == WV &&
                      al16(kbase) && al16(vbase) &&
                      al16(knb) && al16(vnb) && (!kProd || (al16(sbase) && al16(kgb))) && (t_begin % 4) == 0;
    auto tile_full = [&](int j) { return t_begin + (int64_t)(j + 1) * kRows <= t_end; };

    auto issue = [&](int j, int s) {  // thread 0 of the warpgroup: tile j into stage s
      const int64_t t0 = t_begin + (int64_t)j * kRows;
      uint32_t* dst = w_stage + s * C::stage_words;
      uint64_t* bar = &bar_st[s];
      mbar_arrive_expect_tx(bar, (uint32_t)(kRows * 4 * (WK + NS + WV + (kProd ? 3 : 2))));
      for (int g0 = 0; g0 < kRows; g0 += seg) {  // one copy per page segment (the whole tile when unpaged)
        const int64_t sl = ph.slot(t0 + g0);
        bulk_load(dst + g0 * WK, kbase + sl * WK, seg * WK * 4, bar);
        if (kProd) bulk_load(dst + C::st_s + g0 * NS, sbase + sl * NS, seg * NS * 4, bar);
        bulk_load(dst + C::st_v + g0 * WV, vbase + sl * WV, seg * WV * 4, bar);
        bulk_load(dst + C::st_kn + g0, knb + sl, seg * 4, bar);
        if (kProd) bulk_load(dst + C::st_kg + g0, kgb + sl, seg * 4, bar);
        bulk_load(dst + C::st_vn + g0, vnb + sl, seg * 4, bar);
      }
    };
    const int nt_w = ntiles;  // this warpgroup's tiles: all of the item's
    const int slot0 = slot;
    uint32_t pend = 0;  // bit s: a copy into stage s is in flight (thread 0 of the warpgroup)
    // the first tiles' copies (the stages are free: the last item's tiles have been read) land
    // while B1 is written
    if (r == 0 && bulk && ok)
      for (int q = 0; q < kStages && q < nt_w; ++q)
        if (tile_full(q)) {
          issue(q, (slot0 + q) % kStages);
          pend |= 1u << ((slot0 + q) % kStages);
        }

    // ---- B1: fp16 K-major, 128-byte swizzle; row g < group: q'_g over K [0, KC);
    //      prod row GMAX + g: (T q')_g over K [KC, KC + 128); all else zero
    for (int idx = r; idx < NB * (C::KBOX * 8); idx += 128) {
      const int row = idx / (C::KBOX * 8), j = idx - row * (C::KBOX * 8);
      float v[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const int k = 8 * j + e;
        float val = 0.f;
        if (k < KC) {
          if (row < group && k < C::NCODE) val = a.ws_q[(row0 + row) * kAttnQS + k];
        } else if (kProd && k < K) {
          if (row >= GMAX && row - GMAX < group) val = a.ws_sq[(row0 + row - GMAX) * 128 + (k - KC)];
        }
        v[e] = val;
      }
      *reinterpret_cast<uint4*>(smem + C::b1_off + w * C::B1_BYTES + sw128_chunk(row, j, C::B_BOX)) =
          Elem<__half>::pack(v);
    }
    fence_proxy_async_smem();  // generic writes of B1, read by the MMAs
    asm volatile("bar.sync %0, 128;" ::"r"(1 + w) : "memory");

    float m_run[GMAX], l_part[GMAX], a128[GMAX];
#pragma unroll
    for (int g = 0; g < GMAX; ++g) {
      m_run[g] = -INFINITY;
      l_part[g] = 0.f;
      a128[g] = 0.f;
    }
    bool mma1_out = false, mma2_out = false;  // committed and not yet waited for
    int i = 0;
    for (; i < nt_w; ++i) {
      const int j = i;
      const int s = (slot0 + i) % kStages;
      const int64_t t0 = t_begin + (int64_t)j * kRows;
      const int rows = (int)(t_end - t0 < (int64_t)kRows ? t_end - t0 : (int64_t)kRows);
      const bool valid = r < rows;
      const bool staged = bulk && tile_full(j);
      if (staged) {
        // a copy whose wait ran out stays pending: the drain below waits for it again
        if (mbar_wait(&bar_st[s], (par_st >> s) & 1u, a.status, lim)) {
          par_st ^= 1u << s;
          pend &= ~(1u << s);
        } else {
          ok = false;
        }
      }
      if (!wg_all(ok, 1 + w)) {
        ok = false;
        break;
      }
      uint32_t kw[WK], sg[NS > 0 ? NS : 1], vw[WV];
      float kn, kg = 0.f, vn;
      if (staged) {
        const uint32_t st = smem_u32(w_stage + s * C::stage_words);
        if constexpr (WK % 4 == 0) {  // 16-byte rows: vector loads (a 32-bit stride of WK words would conflict)
#pragma unroll
          for (int q = 0; q < WK / 4; ++q) {
            const uint4 v = lds_v4(st + (uint32_t)((r * WK + 4 * q) * 4));
            kw[4 * q] = v.x;
            kw[4 * q + 1] = v.y;
            kw[4 * q + 2] = v.z;
            kw[4 * q + 3] = v.w;
          }
        } else {
#pragma unroll
          for (int q = 0; q < WK; ++q) kw[q] = lds_u32(st + (uint32_t)((r * WK + q) * 4));
        }
        if constexpr (kProd) {
          const uint4 v = lds_v4(st + (uint32_t)((C::st_s + r * NS) * 4));
          sg[0] = v.x;
          sg[1] = v.y;
          sg[2] = v.z;
          sg[3] = v.w;
        }
#pragma unroll
        for (int q = 0; q < WV; ++q) vw[q] = lds_u32(st + (uint32_t)((C::st_v + r * WV + q) * 4));
        kn = __uint_as_float(lds_u32(st + (uint32_t)((C::st_kn + r) * 4)));
        if (kProd) kg = __uint_as_float(lds_u32(st + (uint32_t)((C::st_kg + r) * 4)));
        vn = __uint_as_float(lds_u32(st + (uint32_t)((C::st_vn + r) * 4)));
      } else {
        const int64_t sl = valid ? ph.slot(t0 + r) : 0;  // this token's row in its pool
#pragma unroll
        for (int q = 0; q < WK; ++q) kw[q] = valid ? __ldg(kbase + sl * a.ldk + q) : 0u;
        if constexpr (kProd) {
#pragma unroll
          for (int q = 0; q < NS; ++q) sg[q] = valid ? __ldg(sbase + sl * a.lds + q) : 0u;
        }
#pragma unroll
        for (int q = 0; q < WV; ++q) vw[q] = valid ? __ldg(vbase + sl * a.ldv + q) : 0u;
        kn = valid ? __ldg(knb + sl) : 0.f;
        if (kProd) kg = valid ? __ldg(kgb + sl) : 0.f;
        vn = valid ? __ldg(vnb + sl) : 0.f;
      }

      // ---- 1. key -> A1 (tensor memory; MMA1 of the previous tile has completed: its S was read),
      //      16 columns (32 K elements) per tensor-memory store
      {
        constexpr int NCH = (KC / 2 + 15) / 16;
        constexpr int FPH = 16 / DK::EW;  // fields per 16 columns
#pragma unroll
        for (int c = 0; c < NCH; ++c) {
          uint32_t rw[16];
#pragma unroll
          for (int f = 0; f < FPH; ++f) {
            const int fi = c * FPH + f;
            if (fi * DK::P < C::NCODE) {
              const uint32_t v = field<DK::FB, WK>(kw, fi * DK::FB);
              const uint32_t e = klut_l + (v << KL::LSH);
              if constexpr (DK::EW == 4) {
                const uint4 x = lds_v4(e);
                rw[4 * f] = x.x;
                rw[4 * f + 1] = x.y;
                rw[4 * f + 2] = x.z;
                rw[4 * f + 3] = x.w;
              } else if constexpr (DK::EW == 2) {
                const uint2 x = lds_v2(e);
                rw[2 * f] = x.x;
                rw[2 * f + 1] = x.y;
              } else {
                rw[f] = lds_u32(e);
              }
            } else {
#pragma unroll
              for (int q = 0; q < DK::EW; ++q) rw[DK::EW * f + q] = 0u;
            }
#pragma unroll
            for (int q = 0; q < DK::EW; ++q) {  // K elements past the stored codes are zero
              const int k0 = 2 * (16 * c + DK::EW * f + q);
              if (k0 >= C::NCODE) rw[DK::EW * f + q] = 0u;
              else if (k0 + 1 >= C::NCODE) rw[DK::EW * f + q] &= 0xFFFFu;
            }
          }
          if (16 * c + 16 <= KC / 2) tmem_st16(a1_t + (uint32_t)(16 * c), rw);
          else tmem_st8(a1_t + (uint32_t)(16 * c), rw);  // RotorQuant: 72 = 4 x 16 + 8 columns
        }
        if constexpr (kProd) {
#pragma unroll
          for (int c = 0; c < 4; ++c) {  // 32 signs (4 bytes) per 16 columns
            uint32_t rw[16];
#pragma unroll
            for (int bq = 0; bq < 4; ++bq) {
              const uint32_t v = (sg[c] >> (8 * bq)) & 0xFFu;
              const uint4 x = lds_v4(slut_l + (v << 6));
              rw[4 * bq] = x.x;
              rw[4 * bq + 1] = x.y;
              rw[4 * bq + 2] = x.z;
              rw[4 * bq + 3] = x.w;
            }
            tmem_st16(a1_t + (uint32_t)(KC / 2 + 16 * c), rw);
          }
        }
      }
      tmem_wait_st();
      tc_fence_before();
      // every thread has read its stage words: the stage may be refilled
      asm volatile("bar.sync %0, 128;" ::"r"(1 + w) : "memory");
      if (r == 0) {
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < K / 16; ++kk) {
          const uint32_t boff = (uint32_t)((kk >> 2) * C::B_BOX + (kk & 3) * 32);
          umma_f16_ts(s_mma, a1_mma + (uint32_t)(8 * kk), umma_desc_sw128(b1_s + boff, 16, 1024), kId1, kk > 0);
        }
        umma_commit(bar1);
        const int in = i + kStages;
        if (staged && in < nt_w && tile_full(in)) {
          issue(in, s);
          pend |= 1u << s;
        }
      }
      mma1_out = true;

      // ---- 2. value -> A2 (shared memory, MN-major): wait until MMA2 of the previous tile is done
      if (mma2_out) {
        ok = mbar_wait(bar2, n2 & 1u, a.status) && ok;
        ++n2;
        mma2_out = false;
      }
      float c128;
      {
        constexpr int FPCH = 8 / DV::P;  // fields per 16-byte chunk (8 coordinates)
#pragma unroll
        for (int at = 0; at < 2; ++at) {
#pragma unroll
          for (int ch = 0; ch < 8; ++ch) {
            uint32_t wv[4];
#pragma unroll
            for (int f = 0; f < FPCH; ++f) {
              const int code0 = 64 * at + 8 * ch + DV::P * f;
              const uint32_t v = field<DV::FB, WV>(vw, code0 * VB);
              const uint32_t e = vlut_l + (v << VL::LSH);
              if constexpr (DV::EW == 4) {
                const uint4 x = lds_v4(e);
                wv[0] = x.x;
                wv[1] = x.y;
                wv[2] = x.z;
                wv[3] = x.w;
              } else if constexpr (DV::EW == 2) {
                const uint2 x = lds_v2(e);
                wv[2 * f] = x.x;
                wv[2 * f + 1] = x.y;
              } else {
                wv[f] = lds_u32(e);
              }
            }
            const uint32_t addr =
                a2_s + (uint32_t)(at * C::A2_ATOM + (r >> 3) * 1024 + (r & 7) * 128 + ((ch ^ (r & 7)) << 4));
            sts_v4(addr, make_uint4(wv[0], wv[1], wv[2], wv[3]));
          }
        }
        c128 = s_vc[field<VB, WV>(vw, 128 * VB)];
      }

      // ---- 3. logits of this tile: wait for MMA1
      ok = mbar_wait(bar1, n1 & 1u, a.status) && ok;
      ++n1;
      mma1_out = false;
      tc_fence_after();
      float sv[NB];
      tmem_ld16(s_t, sv);
      float lg[GMAX];
      const float kqs = a.qjl_scale * kg;
#pragma unroll
      for (int g = 0; g < GMAX; ++g) {
        const float dot = kProd ? fmaf(kqs, sv[GMAX + g], sv[g]) : sv[g];
        lg[g] = (valid && g < group) ? a.scale * kn * dot : -INFINITY;
      }
      // Weights against the running maximum m (lazy rescaling): while every weight stays <= 256 and
      // every w ||v|| <= 8192 (inside fp16) the maximum is left as it is; otherwise (always on the first
      // tile, where m = -inf) the warpgroup forms the exact maximum, rescales what it has accumulated and
      // recomputes the weights. Either way all sums refer to the same m.
      float p[GMAX];
      bool need = false;
#pragma unroll
      for (int g = 0; g < GMAX; ++g) {
        p[g] = (lg[g] == -INFINITY) ? 0.f : __expf(lg[g] - m_run[g]);
        need = need || !(p[g] <= 256.f) || !(p[g] * vn <= 8192.f);
      }
      auto write_b2 = [&]() {
        // weights w_t ||v_t|| as B2 (fp16, K-major: row g, K = token r): neighbouring tokens share a
        // 4-byte word; the even thread of a pair writes the first half of the rows, the odd one the rest
        constexpr int HR = GMAX / 2;
        const bool odd = (r & 1) != 0;
        const int rb = r & ~1;
#pragma unroll
        for (int k = 0; k < HR; ++k) {
          const float lo = p[k] * vn, hi = p[HR + k] * vn;  // compile-time indices: p stays in registers
          const float mine = odd ? hi : lo;
          const float give = odd ? lo : hi;
          const float other = __shfl_xor_sync(0xffffffffu, give, 1);
          const int g = odd ? HR + k : k;
          const __half2 h = odd ? __floats2half2_rn(other, mine) : __floats2half2_rn(mine, other);
          const uint32_t addr = b2_s + (uint32_t)((rb >> 6) * C::B_BOX + g * 128 +
                                                  ((((rb & 63) >> 3) ^ (g & 7)) << 4) + (rb & 7) * 2);
          asm volatile("st.shared.b32 [%0], %1;" ::"r"(addr), "r"(*reinterpret_cast<const uint32_t*>(&h))
                       : "memory");
        }
      };
      write_b2();
      fence_proxy_async_smem();  // A2 and B2 were written by generic stores
      tc_fence_before();
      if (wg_any(need, 1 + w)) {  // (the barrier before MMA2 when no rescaling is needed)
#pragma unroll
        for (int g = 0; g < GMAX; ++g) {
          const float v = warp_max_f32(lg[g]);
          if (lane == 0) red[q4 * GMAX + g] = v;
        }
        asm volatile("bar.sync %0, 128;" ::"r"(1 + w) : "memory");
        float alpha[GMAX];
        bool grew = false;
#pragma unroll
        for (int g = 0; g < GMAX; ++g) {
          const float mx = fmaxf(fmaxf(red[g], red[GMAX + g]), fmaxf(red[2 * GMAX + g], red[3 * GMAX + g]));
          const float m_new = fmaxf(m_run[g], mx);
          alpha[g] = (m_new == m_run[g]) ? 1.f : __expf(m_run[g] - m_new);  // exp(-inf) = 0: nothing yet
          grew = grew || (m_new != m_run[g]);
          p[g] = (lg[g] == -INFINITY) ? 0.f : __expf(lg[g] - m_new);
          m_run[g] = m_new;
          l_part[g] *= alpha[g];
          a128[g] *= alpha[g];
        }
        // the value sums so far (lane r = coordinate r) follow the new maximum
        if (i > 0 && grew) {
          float o[NB];
          tmem_ld16(o_t, o);
          uint32_t ow[NB];
#pragma unroll
          for (int g = 0; g < NB; ++g) ow[g] = __float_as_uint(g < GMAX ? o[g] * alpha[g] : 0.f);
          tmem_st16(o_t, ow);
          tmem_wait_st();
        }
        // every thread has read red and the old B2 words are no longer needed: rewrite them
        write_b2();
        fence_proxy_async_smem();
        tc_fence_before();
        asm volatile("bar.sync %0, 128;" ::"r"(1 + w) : "memory");
      }
#pragma unroll
      for (int g = 0; g < GMAX; ++g) {
        l_part[g] += p[g];
        a128[g] = fmaf(p[g] * vn, c128, a128[g]);
      }
      if (r == 0) {
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kRows / 16; ++kk) {
          const uint32_t aoff = (uint32_t)(kk * 16 * 128);
          const uint32_t boff = (uint32_t)((kk >> 2) * C::B_BOX + (kk & 3) * 32);
          umma_f16(o_mma, umma_desc_sw128(a2_s + aoff, C::A2_ATOM, 1024), umma_desc_sw128(b2_s + boff, 16, 1024),
                   kId2, i > 0 || kk > 0);
        }
        umma_commit(bar2);
      }
      mma2_out = true;
    }

    // ---- this warpgroup's partial of the item: chunk `chunk` of each query row
    const int64_t nck = a.n_chunks;
    const int64_t cidx = chunk;
    float o[NB];
    if (mma2_out) {
      ok = mbar_wait(bar2, n2 & 1u, a.status) && ok;
      ++n2;
      mma2_out = false;
    }
    if (mma1_out) {  // a time-out between MMA1 and its wait
      ok = mbar_wait(bar1, n1 & 1u, a.status) && ok;
      ++n1;
      mma1_out = false;
    }
    // copies still in flight exist only after a time-out broke the tile loop: they land before the
    // warpgroup leaves (it stops after such an item, so the stage parities need no update)
    if (r == 0)
      for (int s2 = 0; s2 < kStages; ++s2)
        if ((pend >> s2) & 1u) {
          mbar_wait(&bar_st[s2], (par_st >> s2) & 1u, a.status);
          ok = false;
        }
    slot = (slot0 + nt_w) % kStages;
    ok = wg_all(ok, 1 + w);  // uniform before the warp-collective tensor-memory load
    tc_fence_after();
    if (i > 0 && ok) {
      tmem_ld16(o_t, o);
#pragma unroll
      for (int g = 0; g < GMAX; ++g)
        if (g < group) a.ws_acc[((row0 + g) * nck + cidx) * kAttnAS + r] = o[g];
    }
#pragma unroll
    for (int g = 0; g < GMAX; ++g) {
      float v = l_part[g], u = a128[g];
#pragma unroll
      for (int of = 16; of > 0; of >>= 1) {
        v += __shfl_xor_sync(0xffffffffu, v, of);
        u += __shfl_xor_sync(0xffffffffu, u, of);
      }
      l_part[g] = v;
      a128[g] = u;
    }
    if (lane == 0)
#pragma unroll
      for (int g = 0; g < GMAX; ++g) red[q4 * GMAX + g] = l_part[g];
    asm volatile("bar.sync %0, 128;" ::"r"(1 + w) : "memory");
    float lsum[GMAX];
#pragma unroll
    for (int g = 0; g < GMAX; ++g) lsum[g] = (red[g] + red[GMAX + g]) + (red[2 * GMAX + g] + red[3 * GMAX + g]);
    asm volatile("bar.sync %0, 128;" ::"r"(1 + w) : "memory");
    if (lane == 0)
#pragma unroll
      for (int g = 0; g < GMAX; ++g) red[q4 * GMAX + g] = a128[g];
    asm volatile("bar.sync %0, 128;" ::"r"(1 + w) : "memory");
#pragma unroll
    for (int g = 0; g < GMAX; ++g) {
      if (g < group && r == g) {
        const int64_t base = (row0 + g) * nck + cidx;
        const float asum = (red[g] + red[GMAX + g]) + (red[2 * GMAX + g] + red[3 * GMAX + g]);
        // a warpgroup without tiles leaves an empty partial: weight zero in the merge
        a.ws_ml[base * 2] = i > 0 ? m_run[g] : -INFINITY;
        a.ws_ml[base * 2 + 1] = lsum[g];
        a.ws_acc[base * kAttnAS + 128] = i > 0 ? asum : 0.f;
      }
    }
    if (i == 0 || !ok)
      for (int g = 0; g < group && g < GMAX; ++g) a.ws_acc[((row0 + g) * nck + cidx) * kAttnAS + r] = 0.f;
    tc_fence_before();
    // the warpgroup is done with its B1, red and this item's buffers; it stops after a time-out
    if (!wg_all(ok, 1 + w)) break;
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <int KM, int KB, int VB>
static cudaError_t launch_t(const AttnArgs& a, cudaStream_t st, int num_sms) {
  using C = Cfg<KM, KB, VB>;
  auto kern = attn_tc_kernel<KM, KB, VB>;
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::alloc);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  const int64_t items = a.n_heads * ((a.n_tokens + a.tokens_per_cta - 1) / a.tokens_per_cta);
  const int64_t grid = items < num_sms ? items : num_sms;
  kern<<<(unsigned)grid, kThreads, C::alloc, st>>>(a);
  return cudaGetLastError();
}

}  // namespace attn_tc

bool attn_tc_supported(int k_method, int k_cbits, int v_bits, int group) {
  if (v_bits != 3) return false;
  switch (k_method) {
    case KVRQ_TQ_PROD: return (k_cbits == 2 || k_cbits == 3) && group <= attn_tc::NB / 2;
    case KVRQ_TQ_MSE: return (k_cbits == 2 || k_cbits == 3 || k_cbits == 4) && group <= attn_tc::NB;
    case KVRQ_RQ_MSE: return (k_cbits == 2 || k_cbits == 3) && group <= attn_tc::NB;
    default: return false;
  }
}

cudaError_t launch_attention_tc(int k_method, int k_cbits, const AttnArgs& a, cudaStream_t st, int num_sms) {
  using namespace attn_tc;
  switch (k_method) {
    case KVRQ_TQ_PROD:
      return k_cbits == 2 ? launch_t<KVRQ_TQ_PROD, 2, 3>(a, st, num_sms) : launch_t<KVRQ_TQ_PROD, 3, 3>(a, st, num_sms);
    case KVRQ_TQ_MSE:
      if (k_cbits == 2) return launch_t<KVRQ_TQ_MSE, 2, 3>(a, st, num_sms);
      if (k_cbits == 3) return launch_t<KVRQ_TQ_MSE, 3, 3>(a, st, num_sms);
      return launch_t<KVRQ_TQ_MSE, 4, 3>(a, st, num_sms);
    default:
      return k_cbits == 2 ? launch_t<KVRQ_RQ_MSE, 2, 3>(a, st, num_sms) : launch_t<KVRQ_RQ_MSE, 3, 3>(a, st, num_sms);
  }
}

}  // namespace kvrq
