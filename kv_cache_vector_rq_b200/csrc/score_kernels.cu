// Attention scores q . k_hat straight from packed keys, on tcgen05 tensor cores.
//
// Method: "TurboQuant 论文解读", "随机旋转（Lemma 1）" -- instead of turning every
// stored key back with Pi^T, rotate the query once (q' = Pi q) and take its
// inner product with the quantized rotated key; "TurboQuant + RotorQuant",
// "How TurboQuant Works" -- <q, k> ~ <q, k_mse> + ||r|| sqrt(pi/2)/m <S q, sign(S r)>;
// its closing note of "When to Use Which" -- speed parity needs Q K^T computed
// directly from the compressed indices. For RotorQuant the same identity holds
// per group: <q, x_hat> = ||x|| sum_g <R_g q_g R_g~, c_hat_g>, q zero-padded.
//
// B200 design. A CTA owns one KV head and a contiguous token range. It rotates
// the head's query group once (Pi q and T Pi q from staged copies of Pi and T,
// or the per-group sandwich) into the MMA B operand (N = 16..64 rows, fp16, in
// shared memory). Keys are then handled in 128-token tiles, the M = 128 rows
// of the MMA, by two or three decode warpgroups that take tiles in turn:
//   * packed code rows and sign rows arrive by bulk copy into a ring of
//     stages per warpgroup; every warpgroup is its own pipeline, its
//     first thread issuing the copies and the MMAs of the warpgroup's tiles;
//   * each thread decodes its key into fp16 operand words through small
//     shared-memory tables (one lookup per 8-bit or 6-bit field of codes, and
//     per byte of signs), replicated per lane so that the lookups of a warp
//     never collide on a bank, and writes them with tcgen05.st straight into
//     its lane of the warpgroup's A region in tensor memory -- the decoded keys
//     never pass through shared memory;
//   * after a warpgroup barrier that thread issues tcgen05.mma with A in
//     tensor memory and B in shared memory into one of the warpgroup's two
//     accumulators;
//   * while the next tile is being decoded the warpgroup reads the previous
//     tile's accumulator row per thread (||k|| and the QJL term) and writes
//     fp32 scores, coalesced across tokens.

#include <cuda_runtime.h>

#include <type_traits>

#include "kvrq_device.cuh"
#include "score_launch.h"
#include "tc_decode.cuh"

namespace kvrq {
namespace score {

constexpr int kRows = 128;                  // tokens per tile (TMEM lanes)
constexpr int kStages = 4;                  // code stages per warpgroup
constexpr uint32_t kTmemCols = 512;

template <int METHOD, int BITS, int NB>
struct Cfg {
  static constexpr bool kProd = METHOD == KVRQ_TQ_PROD;
  static constexpr int D = 128;
  static constexpr int NCODE = METHOD == KVRQ_RQ_MSE ? 129 : 128;  // stored codes per key
  static constexpr int KC = METHOD == KVRQ_RQ_MSE ? 144 : 128;     // MMA K of the centroid part
  static constexpr int K = KC + (kProd ? 128 : 0);                 // total MMA K
  static constexpr int KA = K / 2;                                  // A columns in TMEM (fp16 pairs)
  static constexpr int KAP = (KA + 31) / 32 * 32;                   // A region, 32-column aligned
  static constexpr int KBOX = (K + 63) / 64;                        // 64-element B boxes per row
  static constexpr int W = (NCODE * BITS + 31) / 32;                // code words per key
  static constexpr int NS = kProd ? 4 : 0;                          // sign words per key (m = 128)
  static constexpr int B_BOX = NB * 128;
  static constexpr int QS = D + 16;                                 // row stride of the query scratch
  static constexpr int MS = 130;                                    // padded row (halves) of a staged matrix
  // TMEM columns per warpgroup: A, then two accumulators; as many decode
  // warpgroups (up to three) as tensor memory holds
  static constexpr int WCOLS = (KAP + 2 * NB + 31) / 32 * 32;
  static constexpr int kNWG = 3 * WCOLS <= (int)kTmemCols ? 3 : 2;
  static constexpr int kThreads = kNWG * 128;
  static_assert(kNWG * WCOLS <= (int)kTmemCols, "tensor memory");
  // shared memory; a stage holds a tile's code rows and sign rows
  static constexpr int stage_words = kRows * (W + NS);
  static constexpr int lut_bytes = Dec<BITS>::BYTES;
  static constexpr int slut_bytes = kProd ? 256 * 128 : 0;  // byte of signs -> 8 x (+1/-1), 8 replicas
  static constexpr int lut_off = 0;
  static constexpr int slut_off = lut_off + lut_bytes;
  static constexpr int stage_off = slut_off + slut_bytes;
  static constexpr int ring_end = stage_off + kNWG * kStages * stage_words * 4;
  // prologue scratch (rotated queries, staged Pi or T) aliases tables and stages
  static constexpr int q_bytes = 2 * NB * QS * 4;
  static constexpr int m_off = ((q_bytes + 15) / 16) * 16;
  static constexpr int pro_end = m_off + D * MS * 2;
  static constexpr int b_off = (((ring_end > pro_end ? ring_end : pro_end) + 1023) / 1024) * 1024;
  static constexpr int bar_off = b_off + KBOX * B_BOX;
  // barriers: stage full [kNWG][kStages], accumulator full [kNWG][2]
  static constexpr int nbars = kNWG * kStages + 2 * kNWG;
  static constexpr int tmem_off = bar_off + nbars * 8;
  static constexpr int alloc = tmem_off + 16 + 1024;
};

template <int METHOD, int BITS, int NB>
__global__ void __launch_bounds__(Cfg<METHOD, BITS, NB>::kThreads, 1) score_kernel(ScoreArgs a) {
  using C = Cfg<METHOD, BITS, NB>;
  using DC = Dec<BITS>;
  constexpr int D = C::D, K = C::K, KC = C::KC, W = C::W, NS = C::NS;
  constexpr int kNWG = C::kNWG, kThreads = C::kThreads;
  constexpr bool kProd = C::kProd;
  constexpr uint32_t kIdesc = umma_idesc_f16(false, false, false, NB, kRows);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* s_b = smem + C::b_off;
  uint32_t* s_stage = reinterpret_cast<uint32_t*>(smem + C::stage_off);
  const uint8_t* s_lut = smem + C::lut_off;
  const uint8_t* s_slut = smem + C::slut_off;
  float* s_q = reinterpret_cast<float*>(smem);
  uint64_t* s_bar = reinterpret_cast<uint64_t*>(smem + C::bar_off);
  uint64_t* bar_stage = s_bar;                 // [w * kStages + s]
  uint64_t* bar_acc = s_bar + kNWG * kStages;  // [w * 2 + b]
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + C::tmem_off);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = a.group;
  const int64_t head = blockIdx.y;
  const int64_t t_begin = (int64_t)blockIdx.x * a.tokens_per_cta;
  const PagedHead ph = paged_head(head, a.n_tokens, a.block_tables, a.ld_table, a.seq_lens, a.page_tokens, a.n_seqs,
                                  a.kv_heads);
  const int64_t t_end = ph.n_tokens < t_begin + a.tokens_per_cta ? ph.n_tokens : t_begin + a.tokens_per_cta;
  const int ntiles = t_end > t_begin ? (int)((t_end - t_begin + kRows - 1) / kRows) : 0;
  const uint32_t* codes_h = a.codes + ph.pool_head * a.codes_head_stride;
  const uint32_t* signs_h = kProd ? a.signs + ph.pool_head * a.signs_head_stride : nullptr;
  const float* norms_h = a.norms + ph.pool_head * a.tok_head_stride;
  const float* gammas_h = kProd ? a.gammas + ph.pool_head * a.tok_head_stride : nullptr;
  // a paged tile is copied one page segment (min(page, 128) rows) at a time: pages of a power of two >= 16
  // slots start 16-byte aligned and split a 128-token tile evenly
  const int seg = !ph.table ? kRows : (ph.ptok < kRows ? ph.ptok : kRows);
  const bool seg_ok = !ph.table || (ph.shift >= 4);
  // code rows of a tile are one contiguous, 16-byte aligned block when unpadded
  const bool bulk = seg_ok && a.ldc == W && (!kProd || a.lds == NS) && ((reinterpret_cast<uintptr_t>(codes_h) & 15) == 0) &&
                    (!kProd || (reinterpret_cast<uintptr_t>(signs_h) & 15) == 0) && ((kRows * W * 4) % 16 == 0);
  auto tile_full = [&](int j) { return t_begin + (int64_t)(j + 1) * kRows <= t_end; };
  const uint32_t lim = a.spin_limit < 0 ? kSpinLimit : (uint32_t)a.spin_limit;  // main loop (the drain: default)

  if (tid == 0) {
    for (int s = 0; s < C::nbars; ++s) mbar_init(&s_bar[s], 1);
    fence_barrier_init();
  }
  if (warp == 0) tmem_alloc(s_tmem, kTmemCols);

  // ---------------------------------------------------------------- rotated queries
  // s_q rows [0, G): q' (fp32); rows [NB, NB + G): the raw queries, later (T q')
  const int Gp = kProd ? NB / 2 : NB;  // B rows of the centroid part
  for (int idx = tid; idx < G * D; idx += kThreads) {
    const int g = idx / D, i = idx - g * D;
    float v = 0.f;
    const int64_t qrow = (head * G + g) * a.ldq;
    if (a.q_f32) v = reinterpret_cast<const float*>(a.q)[qrow + i];
    else if (a.q_bf16) v = __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(a.q)[qrow + i]);
    else v = __half2float(reinterpret_cast<const __half*>(a.q)[qrow + i]);
    s_q[(NB + g) * C::QS + i] = v;
  }
  __syncthreads();
  if (METHOD == KVRQ_RQ_MSE) {
    // per group: y = M q_g (zero pad beyond d), 3G = 129 coordinates
    for (int idx = tid; idx < G * 43; idx += kThreads) {
      const int g = idx / 43, grp = idx - g * 43;
      const float4 r = __ldg(reinterpret_cast<const float4*>(a.rotors) + grp);
      float m[9];
      rotor_matrix(r.x, r.y, r.z, r.w, m);
      const float* qr = s_q + (NB + g) * C::QS;
      float v[3];
#pragma unroll
      for (int i = 0; i < 3; ++i) v[i] = (3 * grp + i < D) ? qr[3 * grp + i] : 0.f;
#pragma unroll
      for (int i = 0; i < 3; ++i)
        s_q[g * C::QS + 3 * grp + i] = fmaf(m[3 * i + 2], v[2], fmaf(m[3 * i + 1], v[1], m[3 * i] * v[0]));
    }
  } else {
    // q' = Pi q: Pi staged in shared memory (coalesced 16-byte loads, padded rows), then
    // out[g][i] = sum_k M[i][k] vec[g][k] with one (g, i) per thread and step
    uint16_t* s_m = reinterpret_cast<uint16_t*>(smem + C::m_off);
    auto stage = [&](const void* src) {
      const uint4* g = reinterpret_cast<const uint4*>(src);
      for (int i = tid; i < D * D / 8; i += kThreads) {
        const uint4 v = __ldg(g + i);
        uint32_t* d32 = reinterpret_cast<uint32_t*>(s_m + (i / 16) * C::MS + (i % 16) * 8);
        d32[0] = v.x;
        d32[1] = v.y;
        d32[2] = v.z;
        d32[3] = v.w;
      }
    };
    auto mat_vec = [&](bool bf16, const float* vec_base, float* out_base) {
      for (int idx = tid; idx < G * D; idx += kThreads) {
        const int g = idx / D, i = idx - g * D;
        const uint32_t* row = reinterpret_cast<const uint32_t*>(s_m + i * C::MS);
        const float* vec = vec_base + g * C::QS;
        float acc0 = 0.f, acc1 = 0.f;
#pragma unroll 8
        for (int k = 0; k < D; k += 2) {
          const uint32_t w = row[k / 2];
          float p0, p1;
          if (bf16) {
            p0 = __uint_as_float(w << 16);
            p1 = __uint_as_float(w & 0xFFFF0000u);
          } else {
            const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w));
            p0 = f.x;
            p1 = f.y;
          }
          const float2 qv = *reinterpret_cast<const float2*>(vec + k);
          acc0 = fmaf(p0, qv.x, acc0);
          acc1 = fmaf(p1, qv.y, acc1);
        }
        out_base[g * C::QS + i] = acc0 + acc1;
      }
    };
    stage(a.pi);
    __syncthreads();
    mat_vec(a.pi_bf16, s_q + NB * C::QS, s_q);
    __syncthreads();
    if (kProd) {
      stage(a.T);
      __syncthreads();
      mat_vec(false, s_q, s_q + NB * C::QS);
    }
  }
  __syncthreads();
  // B operand [NB rows][K] fp16, 128-byte swizzled, K-major: row g < G holds q'_g over the
  // centroid part; for prod row Gp + g holds (T q')_g over the sign part; all else zero.
  for (int idx = tid; idx < NB * (C::KBOX * 8); idx += kThreads) {
    const int row = idx / (C::KBOX * 8), j = idx - row * (C::KBOX * 8);  // 16-byte chunk j of the row
    float v[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int k = 8 * j + e;
      float val = 0.f;
      if (k < KC) {
        if (row < G && k < (METHOD == KVRQ_RQ_MSE ? 129 : D)) val = s_q[row * C::QS + k];
      } else if (kProd && k < K) {
        if (row >= Gp && row - Gp < G) val = s_q[(NB + row - Gp) * C::QS + (k - KC)];
      }
      v[e] = val;
    }
    *reinterpret_cast<uint4*>(s_b + sw128_chunk(row, j, C::B_BOX)) = Elem<__half>::pack(v);
  }
  __syncthreads();  // the prologue scratch (aliasing the tables and stages) has been read

  // ---------------------------------------------------------------- decode tables
  {
    const float* cb = a.centroids;
    // 16-bit slot s of entry e: replica s / P, code j = s % P of the field
    for (int i = tid; i < DC::ENT * 64; i += kThreads) {
      const int e = i >> 6, j = (i & 63) % DC::P;
      reinterpret_cast<__half*>(smem + C::lut_off)[i] = __float2half_rn(cb[(e >> (j * BITS)) & ((1 << BITS) - 1)]);
    }
    if (kProd)
      for (int i = tid; i < 256 * 64; i += kThreads) {
        const int e = i >> 6, j = (i & 63) % 8;
        reinterpret_cast<__half*>(smem + C::slut_off)[i] = __float2half_rn(((e >> j) & 1) ? 1.f : -1.f);
      }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;
  const uint32_t b_s = smem_u32(s_b);

  {
    // ------------------------------------------------------------ decode warpgroups
    const int w = warp >> 2;  // warpgroup
    const int r = tid & 127;  // key row of the tile = TMEM lane
    // The warpgroup is its own pipeline: its thread 0 issues the bulk copies of
    // the warpgroup's tiles and, once all 128 rows are in tensor memory, the MMAs.
    auto issue_stage = [&](int j) {  // thread 0 of the warpgroup
      const int i = j / kNWG, s = i % kStages;
      const int64_t t0 = t_begin + (int64_t)j * kRows;
      uint32_t* dst = s_stage + (w * kStages + s) * C::stage_words;
      uint64_t* bar = &bar_stage[w * kStages + s];
      mbar_arrive_expect_tx(bar, C::stage_words * 4);
      for (int g0 = 0; g0 < kRows; g0 += seg) {  // one copy per page segment (the whole tile when unpaged)
        const int64_t sl = ph.slot(t0 + g0);
        bulk_load(dst + g0 * W, codes_h + sl * W, seg * W * 4, bar);
        if (kProd) bulk_load(dst + kRows * W + g0 * NS, signs_h + sl * NS, seg * NS * 4, bar);
      }
    };
    if (r == 0 && bulk)
      for (int i = 0; i < kStages; ++i) {
        const int j = w + i * kNWG;
        if (j < ntiles && tile_full(j)) issue_stage(j);
      }
    const uint32_t a_mma = tmem + (uint32_t)(w * C::WCOLS);  // lane 0 of the warpgroup's A region
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t a_t = tmem + lane_off + (uint32_t)(w * C::WCOLS);
    const uint32_t acc_t = a_t + (uint32_t)C::KAP;
    const uint32_t lut_l = smem_u32(s_lut) + (uint32_t)((lane % DC::R) * DC::EB);  // this lane's replica
    const uint32_t slut_l = smem_u32(s_slut) + (uint32_t)((lane & 7) * 16);
    bool ok = true;
    float prev_n = 0.f, prev_g = 0.f;

    auto epilogue = [&](int jp, int ip, float nrm, float gam) {
      const int64_t t0 = t_begin + (int64_t)jp * kRows;
      const int rows = (int)(t_end - t0 < (int64_t)kRows ? t_end - t0 : (int64_t)kRows);
      float acc[NB];
#pragma unroll
      for (int c = 0; c < NB / 16; ++c) tmem_ld16(acc_t + (uint32_t)((ip & 1) * NB + 16 * c), &acc[16 * c]);
      if (r < rows) {
        const float qs = a.qjl_scale * gam;
        const int64_t t = t0 + r;
#pragma unroll
        for (int g = 0; g < (kProd ? NB / 2 : NB); ++g) {
          if (g < G) {
            float s = acc[g];
            if (kProd) s = fmaf(qs, acc[NB / 2 + g], s);
            a.scores[(head * G + g) * a.ld_scores + t] = nrm * s;
          }
        }
      }
    };

    constexpr int NCC = (KC / 2 + 15) / 16;  // 16-word chunks of the centroid part
    auto centroid_chunk = [&](int c, const uint32_t (&wc)[W]) {
      uint32_t rw[16];
      constexpr int FPC = 32 / DC::P;  // fields per 16 words
#pragma unroll
      for (int f = 0; f < FPC; ++f) {
        const int fi = c * FPC + f;  // field index: codes fi*P .. fi*P + P - 1
        if (fi * DC::P < C::NCODE) {
          const uint32_t v = field<DC::FB, W>(wc, fi * DC::FB);
          const uint32_t e = lut_l + (v << 7);
          if constexpr (DC::EW == 4) {
            const uint4 x = lds_v4(e);
            rw[4 * f] = x.x;
            rw[4 * f + 1] = x.y;
            rw[4 * f + 2] = x.z;
            rw[4 * f + 3] = x.w;
          } else if constexpr (DC::EW == 2) {
            const uint2 x = lds_v2(e);
            rw[2 * f] = x.x;
            rw[2 * f + 1] = x.y;
          } else {
            rw[f] = lds_u32(e);
          }
        } else {
#pragma unroll
          for (int q = 0; q < DC::EW; ++q) rw[DC::EW * f + q] = 0u;
        }
        // K elements past the stored codes (the RotorQuant tail) are zero
#pragma unroll
        for (int q = 0; q < DC::EW; ++q) {
          const int k0 = 2 * (16 * c + DC::EW * f + q);  // first K element of this word
          if (k0 >= C::NCODE) rw[DC::EW * f + q] = 0u;
          else if (k0 + 1 >= C::NCODE) rw[DC::EW * f + q] &= 0xFFFFu;
        }
      }
      if (16 * c + 16 <= KC / 2) tmem_st16(a_t + (uint32_t)(16 * c), rw);
      else tmem_st8(a_t + (uint32_t)(16 * c), rw);  // RotorQuant: 72 = 4 x 16 + 8 words
    };
    auto sign_chunk = [&](int c, const uint32_t (&sg)[NS > 0 ? NS : 1]) {  // 16 words: 4 bytes of signs
      uint32_t rw[16];
#pragma unroll
      for (int bq = 0; bq < 4; ++bq) {
        const int byte = 4 * c + bq;
        const uint32_t v = (sg[byte >> 2] >> (8 * (byte & 3))) & 0xFFu;
        const uint4 x = lds_v4(slut_l + (v << 7));
        rw[4 * bq] = x.x;
        rw[4 * bq + 1] = x.y;
        rw[4 * bq + 2] = x.z;
        rw[4 * bq + 3] = x.w;
      }
      tmem_st16(a_t + (uint32_t)(KC / 2 + 16 * c), rw);
    };
    auto mma_steps = [&](int i, int k_lo, int k_hi) {  // thread 0 of the warpgroup
      const uint32_t d_t = a_mma + (uint32_t)(C::KAP + (i & 1) * NB);
      for (int kk = k_lo; kk < k_hi; ++kk) {
        const uint32_t boff = (uint32_t)((kk >> 2) * C::B_BOX + (kk & 3) * 32);
        umma_f16_ts(d_t, a_mma + (uint32_t)(8 * kk), umma_desc_sw128(b_s + boff, 16, 1024), kIdesc, kk > 0);
      }
    };

    int i = 0;
    for (int j = w; j < ntiles; j += kNWG, ++i) {
      const int s = i % kStages;
      const int64_t t0 = t_begin + (int64_t)j * kRows;
      const int rows = (int)(t_end - t0 < (int64_t)kRows ? t_end - t0 : (int64_t)kRows);
      // this key's norm and gamma (used by the epilogue one iteration later), packed codes and signs
      const int64_t sl = r < rows ? ph.slot(t0 + r) : 0;  // this key's row in its pool
      const float nrm = r < rows ? __ldg(norms_h + sl) : 0.f;
      const float gam = (kProd && r < rows) ? __ldg(gammas_h + sl) : 0.f;
      uint32_t wc[W], sg[NS > 0 ? NS : 1];
      // both waits of the tile first; the warpgroup leaves together if either ran out
      if (bulk && tile_full(j))
        ok = mbar_wait(&bar_stage[w * kStages + s], (uint32_t)((i / kStages) & 1), a.status, lim);
      if (i > 0) ok = mbar_wait(&bar_acc[w * 2 + ((i - 1) & 1)], (uint32_t)(((i - 1) >> 1) & 1), a.status, lim) && ok;
      if (!wg_all(ok, 1 + w)) {
        ok = false;
        break;
      }
      if (bulk && tile_full(j)) {
        const uint32_t* stg = s_stage + (w * kStages + s) * C::stage_words;
        const uint32_t stg_a = smem_u32(stg);
        if constexpr (W % 4 == 0) {
#pragma unroll
          for (int q = 0; q < W / 4; ++q) {
            const uint4 v = lds_v4(stg_a + (uint32_t)((r * W + 4 * q) * 4));
            wc[4 * q] = v.x;
            wc[4 * q + 1] = v.y;
            wc[4 * q + 2] = v.z;
            wc[4 * q + 3] = v.w;
          }
        } else {
#pragma unroll
          for (int q = 0; q < W; ++q) wc[q] = lds_u32(stg_a + (uint32_t)((r * W + q) * 4));
        }
        if constexpr (kProd) {
          const uint4 v = lds_v4(stg_a + (uint32_t)((kRows * W + r * NS) * 4));
          sg[0] = v.x;
          sg[1] = v.y;
          sg[2] = v.z;
          sg[3] = v.w;
        }
      } else {
#pragma unroll
        for (int q = 0; q < W; ++q) wc[q] = r < rows ? __ldg(codes_h + sl * a.ldc + q) : 0u;
        if constexpr (kProd) {
#pragma unroll
          for (int q = 0; q < NS; ++q) sg[q] = r < rows ? __ldg(signs_h + sl * a.lds + q) : 0u;
        }
      }
      // the previous tile's MMA has finished with A: its scores, then this tile's decode
      if (i > 0) {
        tc_fence_after();
        epilogue(j - kNWG, i - 1, prev_n, prev_g);
      }
#pragma unroll
      for (int c = 0; c < NCC; ++c) centroid_chunk(c, wc);
      if constexpr (kProd) {
#pragma unroll
        for (int c = 0; c < 4; ++c) sign_chunk(c, sg);
      }
      prev_n = nrm;  // the loads have long landed by now
      prev_g = gam;
      tmem_wait_st();
      tc_fence_before();
      // All rows of the tile are in tensor memory, and every thread has read its stage: the words it
      // loaded were decoded into the values just stored to tensor memory, so those loads have returned
      // before the barrier that lets the leader refill the stage.
      asm volatile("bar.sync %0, 128;" ::"r"(1 + w) : "memory");
      if (r == 0) {
        tc_fence_after();
        mma_steps(i, 0, K / 16);
        umma_commit(&bar_acc[w * 2 + (i & 1)]);
        const int jn = j + kStages * kNWG;
        if (bulk && jn < ntiles && tile_full(jn)) issue_stage(jn);
      }
    }
    // the last tile of this warpgroup (also waits for its last MMA before TMEM is released)
    if (ok && i > 0) {
      const int jl = w + (i - 1) * kNWG;
      if (mbar_wait(&bar_acc[w * 2 + ((i - 1) & 1)], (uint32_t)(((i - 1) >> 1) & 1), a.status)) {
        tc_fence_after();
        epilogue(jl, i - 1, prev_n, prev_g);
      }
    } else if (!ok && r == 0) {
      // a wait ran out: the MMAs and copies still in flight finish before the CTA exits
      if (i > 0) mbar_wait(&bar_acc[w * 2 + ((i - 1) & 1)], (uint32_t)(((i - 1) >> 1) & 1), a.status);
      for (int s2 = 0; s2 < kStages; ++s2) {
        const int iu = i + s2;  // stages possibly still filling
        if (bulk && w + iu * kNWG < ntiles && tile_full(w + iu * kNWG))
          mbar_wait(&bar_stage[w * kStages + (iu % kStages)], (uint32_t)((iu / kStages) & 1), a.status);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace score

template <int METHOD, int BITS, int NB>
static cudaError_t launch_score_t(const ScoreArgs& a, cudaStream_t st) {
  using C = score::Cfg<METHOD, BITS, NB>;
  auto kern = score::score_kernel<METHOD, BITS, NB>;
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::alloc);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  dim3 grid((unsigned)((a.n_tokens + a.tokens_per_cta - 1) / a.tokens_per_cta), (unsigned)a.n_heads);
  kern<<<grid, C::kThreads, C::alloc, st>>>(a);
  return cudaGetLastError();
}

template <int METHOD, int NB>
static cudaError_t score_by_bits(int cbits, const ScoreArgs& a, cudaStream_t st) {
  switch (cbits) {
    case 1: return launch_score_t<METHOD, 1, NB>(a, st);
    case 2: return launch_score_t<METHOD, 2, NB>(a, st);
    case 3: return launch_score_t<METHOD, 3, NB>(a, st);
    default: return launch_score_t<METHOD, 4, NB>(a, st);
  }
}

template <int METHOD>
static cudaError_t score_by_nb(int nb, int cbits, const ScoreArgs& a, cudaStream_t st) {
  switch (nb) {
    case 16: return score_by_bits<METHOD, 16>(cbits, a, st);
    case 32: return score_by_bits<METHOD, 32>(cbits, a, st);
    default: return score_by_bits<METHOD, 64>(cbits, a, st);
  }
}

cudaError_t launch_score(int method, int nb, int cbits, const ScoreArgs& a, cudaStream_t st) {
  switch (method) {
    case KVRQ_RQ_MSE: return score_by_nb<KVRQ_RQ_MSE>(nb, cbits, a, st);
    case KVRQ_TQ_MSE: return score_by_nb<KVRQ_TQ_MSE>(nb, cbits, a, st);
    default: return score_by_nb<KVRQ_TQ_PROD>(nb, cbits, a, st);
  }
}

}  // namespace kvrq
