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
// B200 design: a CTA owns one KV head and a contiguous token range. It rotates
// the head's query group once (Pi q and T Pi q, or the per-group sandwich) and
// writes it as the MMA B operand (N = 16.. rows, fp16). Then, per 128-token
// tile: packed code rows arrive by bulk copy (double-buffered), each thread
// decodes one token through small shared-memory tables (several codes per
// lookup) into a 128-byte-swizzled fp16 A tile (centroids, then +1/-1 signs for
// TurboQuant-prod), one thread issues tcgen05.mma (M = 128 tokens), and the
// epilogue reads one TMEM lane per token, applies ||k|| (and the QJL term) and
// writes fp32 scores coalesced across tokens.

#include <cuda_runtime.h>

#include <type_traits>

#include "kvrq_device.cuh"
#include "score_launch.h"

namespace kvrq {
namespace score {

constexpr int kRows = 128;  // tokens per tile = threads per CTA

// Codes per lookup for a stored code width b: the table maps a field of
// kPer * b bits to kPer fp16 centroids.
template <int BITS>
struct Dec {
  static constexpr int kPer = BITS == 1 ? 8 : BITS == 2 ? 4 : 2;
  static constexpr int kFieldBits = kPer * BITS;      // 8, 8, 6, 8
  static constexpr int kEntries = 1 << kFieldBits;    // 256, 256, 64, 256
  static constexpr int kEntryBytes = kPer * 2;        // 16, 8, 4, 4
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
  static constexpr int B_BOX = NB * 128;                            // B: box of NB rows
  static constexpr int QS = D + 16;                                 // row stride of the query scratch
  static constexpr int q_bytes = 2 * NB * QS * 4;                   // fp32 rotated queries (prologue only)
  static constexpr int a_bytes = KBOX * A_BOX > q_bytes ? KBOX * A_BOX : q_bytes;
  static constexpr int a_off = 0;                                   // the query scratch aliases the A tile
  static constexpr int q_off = 0;
  static constexpr int b_off = a_off + ((a_bytes + 1023) / 1024) * 1024;
  static constexpr int stage_words = ((kRows * (W + NS) + 3) / 4) * 4;  // codes then signs, per tile
  static constexpr int stage_off = b_off + KBOX * B_BOX;
  static constexpr int lut_off = stage_off + 2 * stage_words * 4;
  static constexpr int lut_bytes = Dec<BITS>::kEntries * Dec<BITS>::kEntryBytes;
  static constexpr int slut_off = lut_off + lut_bytes;  // sign table: byte -> 8 x (+1/-1)
  static constexpr int slut_bytes = kProd ? 256 * 16 : 0;
  static constexpr int bar_off = slut_off + slut_bytes;
  static constexpr int tmem_off = bar_off + 4 * 8;
  static constexpr int bytes = tmem_off + 16;
  static constexpr int alloc = bytes + 1024;
  static constexpr uint32_t kNcols = NB < 32 ? 32 : NB;
};

template <int METHOD, int BITS, int NB>
__global__ void __launch_bounds__(kRows, 1) score_kernel(ScoreArgs a) {
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
  float* s_q = reinterpret_cast<float*>(smem + C::q_off);
  uint64_t* s_bar = reinterpret_cast<uint64_t*>(smem + C::bar_off);  // [0,1] code stages, [2] mma
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + C::tmem_off);

  const int tid = threadIdx.x, warp = tid >> 5;
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
    for (int s = 0; s < 3; ++s) mbar_init(&s_bar[s], 1);
    fence_barrier_init();
  }
  if (warp == 0) tmem_alloc(s_tmem, C::kNcols);

  // ---------------------------------------------------------------- decode tables
  {
    const float* cb = a.centroids;
    for (int e = tid; e < DC::kEntries; e += kRows) {
      __half h[DC::kPer];
#pragma unroll
      for (int j = 0; j < DC::kPer; ++j) h[j] = __float2half_rn(cb[(e >> (j * BITS)) & ((1 << BITS) - 1)]);
#pragma unroll
      for (int j = 0; j < DC::kPer; ++j) reinterpret_cast<__half*>(s_lut + e * DC::kEntryBytes)[j] = h[j];
    }
    if (kProd)
      for (int e = tid; e < 256; e += kRows)
#pragma unroll
        for (int j = 0; j < 8; ++j)
          reinterpret_cast<__half*>(s_slut + e * 16)[j] = __float2half_rn(((e >> j) & 1) ? 1.f : -1.f);
  }

  // ---------------------------------------------------------------- rotated queries
  // s_q[g][i] (fp32): q' = rotated query g; for prod also s_q[G + g][j] = (T q')_j
  const int Gp = kProd ? NB / 2 : NB;  // B rows per part
  for (int idx = tid; idx < G * D; idx += kRows) {
    const int g = idx / D, i = idx - g * D;
    float v = 0.f;
    const int64_t qrow = (head * G + g) * a.ldq;
    if (a.q_f32) v = reinterpret_cast<const float*>(a.q)[qrow + i];
    else if (a.q_bf16) v = __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(a.q)[qrow + i]);
    else v = __half2float(reinterpret_cast<const __half*>(a.q)[qrow + i]);
    s_q[(NB + g) * C::QS + i] = v;  // raw query in the spare rows
  }
  __syncthreads();
  if (METHOD == KVRQ_RQ_MSE) {
    // per group: y = M q_g (zero pad beyond d), 3G = 129 coordinates
    for (int idx = tid; idx < G * 43; idx += kRows) {
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
    // q' = Pi q (row i of Pi times q)
    for (int idx = tid; idx < G * D; idx += kRows) {
      const int g = idx / D, i = idx - g * D;
      const float* qr = s_q + (NB + g) * C::QS;
      float acc = 0.f;
      for (int k = 0; k < D; ++k) {
        const float p = a.pi_bf16 ? __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(a.pi)[i * D + k])
                                  : __half2float(reinterpret_cast<const __half*>(a.pi)[i * D + k]);
        acc = fmaf(p, qr[k], acc);
      }
      s_q[g * C::QS + i] = acc;
    }
  }
  __syncthreads();
  if (kProd) {
    // (T q')_j into the spare rows (the raw queries are no longer needed)
    for (int idx = tid; idx < G * D; idx += kRows) {
      const int g = idx / D, j = idx - g * D;
      const float* qp = s_q + g * C::QS;
      float acc = 0.f;
      for (int k = 0; k < D; ++k) acc = fmaf(__half2float(reinterpret_cast<const __half*>(a.T)[j * D + k]), qp[k], acc);
      s_q[(NB + g) * C::QS + j] = acc;
    }
    __syncthreads();
  }
  // B operand [NB rows][K] fp16, 128-byte swizzled, K-major: row g < G holds q'_g over the
  // centroid part; for prod row Gp + g holds (T q')_g over the sign part; all else zero.
  for (int idx = tid; idx < NB * (C::KBOX * 8); idx += kRows) {
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
  __syncthreads();  // the query scratch (aliasing the A tile) has been read
  // zero the A tile once (its unused K columns stay zero)
  for (int i = tid; i < C::KBOX * C::A_BOX / 16; i += kRows) reinterpret_cast<uint4*>(s_a)[i] = make_uint4(0, 0, 0, 0);
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;
  const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
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
    for (int it = 0; it < 2 && it < ntiles; ++it)
      if (tile_full(it)) issue_stage(it, it);

  bool ok = true;
  for (int it = 0; it < ntiles; ++it) {
    const int st = it & 1;
    const int64_t t0 = t_begin + (int64_t)it * kRows;
    const int rows = (int)(t_end - t0 < (int64_t)kRows ? t_end - t0 : (int64_t)kRows);
    const int64_t t = t0 + tid;
    uint32_t* stg = s_stage + st * C::stage_words;
    const float nrm = tid < rows ? __ldg(norms_h + t) : 0.f;
    const float gam = (kProd && tid < rows) ? __ldg(gammas_h + t) : 0.f;
    if (bulk && tile_full(it)) {
      ok = mbar_wait(&s_bar[st], (par >> st) & 1, a.status);
      par ^= 1u << st;
    } else {
      for (int i = tid; i < rows * W; i += kRows) {
        const int r = i / W, w = i - r * W;
        stg[i] = __ldg(codes_h + (t0 + r) * a.ldc + w);
      }
      if (kProd)
        for (int i = tid; i < rows * NS; i += kRows) {
          const int r = i / NS, w = i - r * NS;
          stg[kRows * W + i] = __ldg(signs_h + (t0 + r) * a.lds + w);
        }
      for (int i = rows * W + tid; i < kRows * W; i += kRows) stg[i] = 0u;  // ragged tail: decode zeros
    }
    if (!__syncthreads_and(ok)) break;

    // ------------------------------------------------------------ decode this thread's key
    uint32_t wc[W];
#pragma unroll
    for (int w = 0; w < W; ++w) wc[w] = stg[tid * W + w];
    {
      // fields of P codes -> P fp16 centroids (P/2 words); codes past the stored ones are zero
      constexpr int P = DC::kPer, FB = DC::kFieldBits;
      constexpr int NF = (C::NCODE + P - 1) / P;
      uint32_t rw[KC / 2];
#pragma unroll
      for (int k = 0; k < KC / 2; ++k) rw[k] = 0u;
#pragma unroll
      for (int f = 0; f < NF; ++f) {
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
      for (int j = 0; j < KC / 8; ++j)
        *reinterpret_cast<uint4*>(s_a + sw128_chunk(tid, j, C::A_BOX)) =
            make_uint4(rw[4 * j], rw[4 * j + 1], rw[4 * j + 2], rw[4 * j + 3]);
    }
    if constexpr (kProd) {
#pragma unroll
      for (int w = 0; w < NS; ++w) {
        const uint32_t sw = stg[kRows * W + tid * NS + w];
#pragma unroll
        for (int bt = 0; bt < 4; ++bt) {
          const uint4 e = *reinterpret_cast<const uint4*>(s_slut + ((sw >> (8 * bt)) & 0xFF) * 16);
          *reinterpret_cast<uint4*>(s_a + sw128_chunk(tid, KC / 8 + w * 4 + bt, C::A_BOX)) = e;
        }
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {
      // refill this code stage two tiles ahead (every thread has read it)
      if (bulk && it + 2 < ntiles && tile_full(it + 2)) issue_stage(it + 2, st);
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < K / 16; ++kk) {
        const uint32_t off = (uint32_t)((kk >> 2) * C::A_BOX + (kk & 3) * 32);
        const uint32_t boff = (uint32_t)((kk >> 2) * C::B_BOX + (kk & 3) * 32);
        umma_f16(tmem, umma_desc_sw128(a_s + off, 16, 1024), umma_desc_sw128(b_s + boff, 16, 1024), kIdesc, kk > 0);
      }
      umma_commit(&s_bar[2]);
    }
    ok = mbar_wait(&s_bar[2], (par >> 2) & 1, a.status) && ok;
    par ^= 4u;
    tc_fence_after();

    // ------------------------------------------------------------ epilogue: one token per thread
    float acc[NB];
#pragma unroll
    for (int c = 0; c < NB / 32 + (NB % 32 ? 1 : 0); ++c) {
      float v[32];
      tmem_ld32(tmem + lane_off + 32 * c, v);
#pragma unroll
      for (int i = 0; i < 32; ++i)
        if (32 * c + i < NB) acc[32 * c + i] = v[i];
    }
    if (tid < rows) {
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
    tc_fence_before();
    __syncthreads();  // the A tile and TMEM are reused by the next tile
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
  kern<<<grid, score::kRows, C::alloc, st>>>(a);
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
