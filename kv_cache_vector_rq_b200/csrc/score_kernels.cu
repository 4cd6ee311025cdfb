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
// B200 design: a CTA of 256 threads owns one KV head and a contiguous token
// range. It rotates the head's query group once (Pi q and T Pi q from staged
// copies of Pi and T, or the per-group sandwich) into the MMA B operand (N = 16..
// rows, fp16). Then, per 128-token tile: packed code rows arrive by bulk copy
// (a ring of eight tiles in flight); the two warpgroups decode the tile's keys into a
// 128-byte-swizzled fp16 A tile (warpgroup 0 the first half of K, warpgroup 1
// the second: for TurboQuant-prod the centroids and the +1/-1 signs) through
// small shared-memory tables; one thread issues tcgen05.mma (M = 128 tokens)
// into one of two TMEM accumulators; while it runs, warpgroup 1 finishes the
// previous tile (one TMEM lane per token: ||k|| and the QJL term, fp32 scores
// written coalesced across tokens) and both warpgroups decode the next one into
// the other A buffer.

#include <cuda_runtime.h>

#include <type_traits>

#include "kvrq_device.cuh"
#include "score_launch.h"

namespace kvrq {
namespace score {

constexpr int kRows = 128;     // tokens per tile
constexpr int kThreads = 256;  // two warpgroups
constexpr int kStages = 8;     // packed-code tiles in flight per CTA

// Codes per lookup for a stored code width b: the table maps a field of
// kPer * b bits to kPer fp16 centroids.
template <int BITS>
struct Dec {
  static constexpr int kPer = BITS == 1 ? 8 : BITS == 2 ? 4 : 2;
  static constexpr int kFieldBits = kPer * BITS;    // 8, 8, 6, 8
  static constexpr int kEntries = 1 << kFieldBits;  // 256, 256, 64, 256
  static constexpr int kEntryBytes = kPer * 2;      // 16, 8, 4, 4
};

template <int METHOD, int BITS, int NB>
struct Cfg {
  static constexpr bool kProd = METHOD == KVRQ_TQ_PROD;
  static constexpr int D = 128;
  static constexpr int NCODE = METHOD == KVRQ_RQ_MSE ? 129 : 128;  // stored codes per key
  static constexpr int KC = METHOD == KVRQ_RQ_MSE ? 144 : 128;     // MMA K of the centroid part
  static constexpr int K = KC + (kProd ? 128 : 0);                 // total MMA K
  static constexpr int KBOX = (K + 63) / 64;                        // 64-element boxes per row
  static constexpr int W = (NCODE * BITS + 31) / 32;                // code words per key
  static constexpr int NS = kProd ? 4 : 0;                          // sign words per key (m = 128)
  static constexpr int A_BOX = kRows * 128;                         // A: box of 128 rows
  static constexpr int A_BYTES = KBOX * A_BOX;
  static constexpr int B_BOX = NB * 128;                            // B: box of NB rows
  static constexpr int QS = D + 16;                                 // row stride of the query scratch
  static constexpr int q_bytes = 2 * NB * QS * 4;                   // fp32 rotated queries (prologue only)
  static constexpr int MS = 130;                                    // padded row (halves) of a staged matrix
  static constexpr int m_off = ((q_bytes + 15) / 16) * 16;          // staged Pi or T (prologue only)
  static constexpr int pro_bytes = m_off + D * MS * 2;
  static constexpr int a_bytes = 2 * A_BYTES > pro_bytes ? 2 * A_BYTES : pro_bytes;
  static constexpr int a_off = 0;  // two A buffers; the prologue scratch aliases them
  static constexpr int b_off = ((a_bytes + 1023) / 1024) * 1024;
  static constexpr int stage_words = ((kRows * (W + NS) + 3) / 4) * 4;  // codes then signs, per tile
  static constexpr int stage_off = b_off + KBOX * B_BOX;
  static constexpr int lut_off = stage_off + kStages * stage_words * 4;
  static constexpr int lut_bytes = Dec<BITS>::kEntries * Dec<BITS>::kEntryBytes;
  static constexpr int slut_off = lut_off + lut_bytes;  // sign table: byte -> 8 x (+1/-1)
  static constexpr int slut_bytes = kProd ? 256 * 16 : 0;
  static constexpr int bar_off = slut_off + slut_bytes;  // [0, kStages) code stages, then 2 mma buffers
  static constexpr int tmem_off = bar_off + (kStages + 2) * 8;
  static constexpr int bytes = tmem_off + 16;
  static constexpr int alloc = bytes + 1024;
  static constexpr uint32_t kNcols = 2 * NB < 32 ? 32 : 2 * NB;  // two accumulators
  // K columns of the centroid part decoded by warpgroup 0 (the rest by warpgroup 1);
  // for prod warpgroup 0 decodes all centroids and warpgroup 1 the signs
  static constexpr int KSPLIT = kProd ? KC : (KC / 16) * 8;
};

template <int METHOD, int BITS, int NB>
__global__ void __launch_bounds__(kThreads, 1) score_kernel(ScoreArgs a) {
  using C = Cfg<METHOD, BITS, NB>;
  using DC = Dec<BITS>;
  constexpr int D = C::D, K = C::K, KC = C::KC, W = C::W, NS = C::NS;
  constexpr bool kProd = C::kProd;
  constexpr uint32_t kIdesc = umma_idesc_f16(false, false, false, NB, kRows);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* s_a = smem + C::a_off;
  uint8_t* s_b = smem + C::b_off;
  uint32_t* s_stage = reinterpret_cast<uint32_t*>(smem + C::stage_off);
  uint8_t* s_lut = smem + C::lut_off;
  uint8_t* s_slut = smem + C::slut_off;
  float* s_q = reinterpret_cast<float*>(smem);
  uint64_t* s_bar = reinterpret_cast<uint64_t*>(smem + C::bar_off);
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + C::tmem_off);

  const int tid = threadIdx.x, warp = tid >> 5;
  const int wg = tid >> 7, key = tid & 127;  // warpgroup, token within the tile
  const int G = a.group;
  const int64_t head = blockIdx.y;
  const int64_t t_begin = (int64_t)blockIdx.x * a.tokens_per_cta;
  const int64_t t_end = a.n_tokens < t_begin + a.tokens_per_cta ? a.n_tokens : t_begin + a.tokens_per_cta;
  const int ntiles = (int)((t_end - t_begin + kRows - 1) / kRows);
  const uint32_t* codes_h = a.codes + head * a.codes_head_stride;
  const uint32_t* signs_h = kProd ? a.signs + head * a.signs_head_stride : nullptr;
  const float* norms_h = a.norms + head * a.tok_head_stride;
  const float* gammas_h = kProd ? a.gammas + head * a.tok_head_stride : nullptr;
  // code rows of a tile are one contiguous, 16-byte aligned block when unpadded
  const bool bulk = a.ldc == W && (!kProd || a.lds == NS) && ((reinterpret_cast<uintptr_t>(codes_h) & 15) == 0) &&
                    (!kProd || (reinterpret_cast<uintptr_t>(signs_h) & 15) == 0) && ((kRows * W * 4) % 16 == 0);

  if (tid == 0) {
    for (int s = 0; s < kStages + 2; ++s) mbar_init(&s_bar[s], 1);
    fence_barrier_init();
  }
  if (warp == 0) tmem_alloc(s_tmem, C::kNcols);

  // ---------------------------------------------------------------- decode tables
  {
    const float* cb = a.centroids;
    for (int e = tid; e < DC::kEntries; e += kThreads) {
#pragma unroll
      for (int j = 0; j < DC::kPer; ++j)
        reinterpret_cast<__half*>(s_lut + e * DC::kEntryBytes)[j] =
            __float2half_rn(cb[(e >> (j * BITS)) & ((1 << BITS) - 1)]);
    }
    if (kProd)
      for (int e = tid; e < 256; e += kThreads)
#pragma unroll
        for (int j = 0; j < 8; ++j)
          reinterpret_cast<__half*>(s_slut + e * 16)[j] = __float2half_rn(((e >> j) & 1) ? 1.f : -1.f);
  }

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
    // thread i < 128 forms row i of Pi against every query of the group
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
    // out[g][i] = sum_k M[i][k] vec[g][k], one (g, i) per thread and step: a warp covers
    // consecutive i of one g (conflict-free padded rows, broadcast vector)
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
  __syncthreads();  // the prologue scratch (aliasing the A buffers) has been read
  // zero both A buffers once (their unused K columns stay zero)
  for (int i = tid; i < 2 * C::A_BYTES / 16; i += kThreads) reinterpret_cast<uint4*>(s_a)[i] = make_uint4(0, 0, 0, 0);
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;
  const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
  const uint32_t a_s = smem_u32(s_a), b_s = smem_u32(s_b);

  auto tile_full = [&](int it) { return t_begin + (int64_t)(it + 1) * kRows <= t_end; };
  auto issue_stage = [&](int it, int st) {  // thread 0
    const int64_t t0 = t_begin + (int64_t)it * kRows;
    uint32_t* dst = s_stage + st * C::stage_words;
    mbar_arrive_expect_tx(&s_bar[st], kRows * (W + NS) * 4);
    bulk_load(dst, codes_h + t0 * W, kRows * W * 4, &s_bar[st]);
    if (kProd) bulk_load(dst + kRows * W, signs_h + t0 * NS, kRows * NS * 4, &s_bar[st]);
  };
  uint32_t par = 0;  // bit s: parity of the next phase of barrier s
  if (tid == 0 && bulk)
    for (int it = 0; it < kStages && it < ntiles; ++it)
      if (tile_full(it)) issue_stage(it, it);

  // epilogue of tile `pt` (warpgroup 1): scores from accumulator pt & 1
  auto epilogue = [&](int pt, float nrm, float gam) {
    const int64_t t0 = t_begin + (int64_t)pt * kRows;
    const int rows = (int)(t_end - t0 < (int64_t)kRows ? t_end - t0 : (int64_t)kRows);
    const int64_t t = t0 + key;
    // NB columns of accumulator pt & 1 (a multiple of 16; never past the allocation)
    float acc[NB];
#pragma unroll
    for (int c = 0; c < NB / 16; ++c) tmem_ld16(tmem + lane_off + (uint32_t)((pt & 1) * NB) + 16 * c, &acc[16 * c]);
    if (key < rows) {
      const float qs = a.qjl_scale * gam;
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

  bool ok = true;
  float prev_n = 0.f, prev_g = 0.f;  // norm / gamma of this thread's key in the previous tile
  for (int it = 0; it < ntiles; ++it) {
    const int st = it % kStages, ab = it & 1;
    constexpr int MB = kStages;  // first mma-buffer barrier
    const int64_t t0 = t_begin + (int64_t)it * kRows;
    const int rows = (int)(t_end - t0 < (int64_t)kRows ? t_end - t0 : (int64_t)kRows);
    uint32_t* stg = s_stage + st * C::stage_words;
    uint8_t* A = s_a + ab * C::A_BYTES;
    const float nrm = (wg == 1 && key < rows) ? __ldg(norms_h + t0 + key) : 0.f;
    const float gam = (kProd && wg == 1 && key < rows) ? __ldg(gammas_h + t0 + key) : 0.f;
    if (bulk && tile_full(it)) {
      ok = mbar_wait(&s_bar[st], (par >> st) & 1, a.status) && ok;
      par ^= 1u << st;
    } else {
      for (int i = tid; i < rows * W; i += kThreads) {
        const int r = i / W, w = i - r * W;
        stg[i] = __ldg(codes_h + (t0 + r) * a.ldc + w);
      }
      if (kProd)
        for (int i = tid; i < rows * NS; i += kThreads) {
          const int r = i / NS, w = i - r * NS;
          stg[kRows * W + i] = __ldg(signs_h + (t0 + r) * a.lds + w);
        }
      for (int i = rows * W + tid; i < kRows * W; i += kThreads) stg[i] = 0u;  // ragged tail decodes to zero
      if (kProd)
        for (int i = rows * NS + tid; i < kRows * NS; i += kThreads) stg[kRows * W + i] = 0u;
    }
    if (!__syncthreads_and(ok)) break;

    // ------------------------------------------------------------ decode key `key` into A[ab]
    if (!kProd || wg == 0) {
      constexpr int P = DC::kPer, FB = DC::kFieldBits;
      constexpr int NF = (C::NCODE + P - 1) / P;
      uint32_t wc[W];
#pragma unroll
      for (int w = 0; w < W; ++w) wc[w] = stg[key * W + w];
      uint32_t rw[KC / 2];
#pragma unroll
      for (int k = 0; k < KC / 2; ++k) rw[k] = 0u;
      // fields of warpgroup 0 (or, for prod, all) / of warpgroup 1
      const int f_lo = (kProd || wg == 0) ? 0 : C::KSPLIT / P;
      const int f_hi = (kProd || wg == 1) ? NF : C::KSPLIT / P;
#pragma unroll
      for (int f = 0; f < NF; ++f) {
        if (f < f_lo || f >= f_hi) continue;
        const int bit = f * FB, word = bit >> 5, sh = bit & 31;
        uint32_t v = wc[word] >> sh;
        if (sh + FB > 32 && word + 1 < W) v |= wc[word + 1] << (32 - sh);
        v &= (1u << FB) - 1u;
        const uint32_t* e = reinterpret_cast<const uint32_t*>(s_lut + v * DC::kEntryBytes);
        const int valid = C::NCODE - f * P;  // stored codes in this field
#pragma unroll
        for (int k = 0; k < P / 2; ++k) {
          uint32_t wv = e[k];
          if (2 * k >= valid) wv = 0u;
          else if (2 * k + 1 >= valid) wv &= 0xFFFFu;
          rw[f * P / 2 + k] = wv;
        }
      }
#pragma unroll
      for (int j = 0; j < KC / 8; ++j) {
        const bool mine = kProd ? true : (wg == 0 ? (8 * j < C::KSPLIT) : (8 * j >= C::KSPLIT));
        if (mine)
          *reinterpret_cast<uint4*>(A + sw128_chunk(key, j, C::A_BOX)) =
              make_uint4(rw[4 * j], rw[4 * j + 1], rw[4 * j + 2], rw[4 * j + 3]);
      }
    }
    if (kProd && wg == 1) {
      // sign part: each byte of signs -> 8 x (+1/-1) fp16
#pragma unroll
      for (int w = 0; w < NS; ++w) {
        const uint32_t sw = stg[kRows * W + key * NS + w];
#pragma unroll
        for (int bt = 0; bt < 4; ++bt) {
          const uint4 e = *reinterpret_cast<const uint4*>(s_slut + ((sw >> (8 * bt)) & 0xFF) * 16);
          *reinterpret_cast<uint4*>(A + sw128_chunk(key, KC / 8 + w * 4 + bt, C::A_BOX)) = e;
        }
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {
      // refill this code stage kStages tiles ahead (every thread has read it)
      if (bulk && it + kStages < ntiles && tile_full(it + kStages)) issue_stage(it + kStages, st);
      tc_fence_after();
      const uint32_t a_buf = a_s + (uint32_t)(ab * C::A_BYTES);
#pragma unroll
      for (int kk = 0; kk < K / 16; ++kk) {
        const uint32_t off = (uint32_t)((kk >> 2) * C::A_BOX + (kk & 3) * 32);
        const uint32_t boff = (uint32_t)((kk >> 2) * C::B_BOX + (kk & 3) * 32);
        umma_f16(tmem + (uint32_t)(ab * NB), umma_desc_sw128(a_buf + off, 16, 1024),
                 umma_desc_sw128(b_s + boff, 16, 1024), kIdesc, kk > 0);
      }
      umma_commit(&s_bar[MB + ab]);
    }
    // finish the previous tile while this one's MMA runs; its MMA is complete
    // before the next decode overwrites its A buffer
    if (it > 0) {
      ok = mbar_wait(&s_bar[MB + (ab ^ 1)], (par >> (MB + (ab ^ 1))) & 1, a.status) && ok;
      par ^= 1u << (MB + (ab ^ 1));
      tc_fence_after();
      if (wg == 1) epilogue(it - 1, prev_n, prev_g);
    }
    prev_n = nrm;
    prev_g = gam;
    tc_fence_before();
  }
  // the last tile
  if (ok && ntiles > 0) {
    const int lt = ntiles - 1;
    ok = mbar_wait(&s_bar[kStages + (lt & 1)], (par >> (kStages + (lt & 1))) & 1, a.status);
    tc_fence_after();
    if (ok && wg == 1) epilogue(lt, prev_n, prev_g);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, C::kNcols);
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
  kern<<<grid, score::kThreads, C::alloc, st>>>(a);
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
