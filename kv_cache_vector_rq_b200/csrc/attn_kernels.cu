// Decode attention straight from a packed KV cache. Keys are RotorQuant,
// TurboQuant-mse or TurboQuant-prod codes; values are RotorQuant codes:
//   out_(h,g) = sum_t softmax_t(scale * <q_(h,g), k_hat_t>) * v_hat_t
// ["TurboQuant и PolarQuant", "Проблема KV-кэша в трансформерах": the softmax of the
//  query-key products over sqrt(d) weights the values; "TurboQuant + RotorQuant",
//  "When to Use Which": attention computed from the compressed indices]
//
// Three launches, no spin-waits:
//  1. attn_rotate_q_kernel: q' = the per-group rotor sandwich of the zero-padded q
//     (RotorQuant keys, 3G = 129 coordinates) or Pi q (TurboQuant keys), and T q'
//     for prod, once per query row.
//  2. attn_chunk_kernel: one CTA per (token chunk, KV head). For each sub-chunk of
//     256 tokens, thread t decodes key t and forms the logits of every query row of
//     the group from q' (the score identity of kv_score_packed); each row's running
//     max and weight sum are updated (online softmax); then thread j accumulates
//     sum_t w_t ||v_t|| c_hat(v_t)_j in the rotated value domain.
//  3. attn_combine_kernel: merges the chunks' (max, sum, accumulator) triples of a
//     query row and applies the inverse sandwich once. x_hat is linear in the
//     rotated codes, so sum_t w_t v_hat_t = M(R_g)^T (sum_t w_t ||v_t|| c_hat(v_t))
//     group by group, and the 43 inverse 3x3 rotations run once per query row
//     instead of once per token.
//
// Both contractions run on the CUDA cores in fp32 (fused multiply-adds of the fp32
// rotated queries with the fp32 centroids; exp and the running sums in fp32).

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "attn_launch.h"
#include "kvrq_device.cuh"

namespace kvrq {
namespace attn {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kGroups = 43;  // rotor groups at d = 128
constexpr int kNcv = 129;    // stored value coordinates (3G)

__device__ __forceinline__ float load_q(const AttnArgs& a, int64_t off) {
  if (a.q_f32) return reinterpret_cast<const float*>(a.q)[off];
  if (a.q_bf16) return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(a.q)[off]);
  return __half2float(reinterpret_cast<const __half*>(a.q)[off]);
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// y = M x for a row-major 128 x 128 matrix M (fp16, or bf16) and x, y in shared memory, by the
// 128 threads of the CTA: warp w takes rows 32w .. 32w + 31. With M 16-byte aligned, lane l reads
// 16 bytes (columns 8 (l mod 16) .. + 7) of rows 32w + 2i + l / 16, i < 16, all sixteen loads issued
// before the first is used; a row's eight-term partial sums are added across its half-warp.
// Otherwise lane l reads columns l, l + 32, l + 64, l + 96 of each row, and the warp adds them.
__device__ __forceinline__ void mat_vec128(const void* M, bool bf16, const float* x, float* y) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if ((reinterpret_cast<uintptr_t>(M) & 15) == 0) {
    const int c0 = 8 * (lane & 15);
    float xv[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) xv[e] = x[c0 + e];
    const uint4* base = reinterpret_cast<const uint4*>(M);
    uint4 w[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) w[i] = __ldg(base + (32 * warp + 2 * i + (lane >> 4)) * 16 + (lane & 15));
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const uint32_t u[4] = {w[i].x, w[i].y, w[i].z, w[i].w};
      float acc = 0.f;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        float2 f;
        if (bf16) f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u[k]));
        else f = __half22float2(*reinterpret_cast<const __half2*>(&u[k]));
        acc = fmaf(f.x, xv[2 * k], acc);
        acc = fmaf(f.y, xv[2 * k + 1], acc);
      }
#pragma unroll
      for (int o = 8; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
      if ((lane & 15) == 0) y[32 * warp + 2 * i + (lane >> 4)] = acc;
    }
    return;
  }
  float xv[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) xv[j] = x[lane + 32 * j];
#pragma unroll 4
  for (int i = 32 * warp; i < 32 * warp + 32; ++i) {
    float acc = 0.f;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int64_t off = (int64_t)i * 128 + lane + 32 * j;
      const float m = bf16 ? __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(M)[off])
                           : __half2float(reinterpret_cast<const __half*>(M)[off]);
      acc = fmaf(m, xv[j], acc);
    }
    acc = warp_sum(acc);
    if (lane == 0) y[i] = acc;
  }
}

// ------------------------------------------------------------------ 1. rotated queries
// One CTA of 128 threads per query row.
__global__ void __launch_bounds__(128) attn_rotate_q_kernel(AttnArgs a, int k_method) {
  __shared__ float s_in[128];
  __shared__ float s_qp[128];
  const int64_t row = blockIdx.x;
  const int tid = threadIdx.x;
  s_in[tid] = load_q(a, row * a.ldq + tid);
  __syncthreads();
  float* wq = a.ws_q + row * kAttnQS;
  if (k_method == KVRQ_RQ_MSE) {
    if (tid < kGroups) {
      const float4 r = __ldg(reinterpret_cast<const float4*>(a.k_rotors) + tid);
      float m[9];
      rotor_matrix(r.x, r.y, r.z, r.w, m);
      float v[3];
#pragma unroll
      for (int i = 0; i < 3; ++i) v[i] = (3 * tid + i < 128) ? s_in[3 * tid + i] : 0.f;
#pragma unroll
      for (int i = 0; i < 3; ++i) wq[3 * tid + i] = fmaf(m[3 * i + 2], v[2], fmaf(m[3 * i + 1], v[1], m[3 * i] * v[0]));
    } else if (tid < kGroups + kAttnQS - 3 * kGroups) {
      wq[3 * kGroups + (tid - kGroups)] = 0.f;
    }
    return;
  }
  // q' = Pi q, then (prod) T q'
  mat_vec128(a.pi, a.pi_bf16, s_in, s_qp);
  __syncthreads();
  wq[tid] = s_qp[tid];
  if (tid < kAttnQS - 128) wq[128 + tid] = 0.f;
  if (k_method != KVRQ_TQ_PROD) return;
  mat_vec128(a.T, false, s_qp, s_in);  // s_in is no longer read: it takes T q'
  __syncthreads();
  a.ws_sq[row * 128 + tid] = s_in[tid];
}

// ------------------------------------------------------------------ 2. chunk partials
// METHOD: the keys' kvrq_method; KCB: stored key-code width; GM: query rows held per
// CTA (8 or 16, >= group; rows >= group carry zero queries and are never written).
template <int METHOD, int KCB, int GM>
__global__ void __launch_bounds__(kThreads) attn_chunk_kernel(AttnArgs a) {
  constexpr bool kProd = METHOD == KVRQ_TQ_PROD;
  constexpr int NCK = METHOD == KVRQ_RQ_MSE ? 3 * kGroups : 128;  // stored key coordinates
  constexpr int KW = (NCK * KCB + 31) / 32;                       // key code words
  constexpr int RPW = GM / kWarps;                                // softmax rows per warp
  static_assert(GM % 8 == 0 && RPW >= 1, "GM is a multiple of the warp count");

  __shared__ __align__(16) float s_q[NCK * GM];               // q'[r][j] at [j * GM + r]
  __shared__ __align__(16) float s_sq[kProd ? 128 * GM : 4];  // (T q')[r][j] at [j * GM + r]
  __shared__ __align__(16) float s_p[kAttnSub * GM];          // logit, then weight * ||v||, of (t, r)
  __shared__ float s_vn[kAttnSub];
  __shared__ float s_kc[16], s_vc[16];
  __shared__ float s_alpha[GM];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t head = blockIdx.y;
  const int chunk = blockIdx.x;
  const int group = a.group;
  const int64_t row0 = head * group;

  for (int idx = tid; idx < NCK * GM; idx += kThreads) {
    const int j = idx / GM, r = idx - j * GM;
    s_q[idx] = r < group ? a.ws_q[(row0 + r) * kAttnQS + j] : 0.f;
  }
  if (kProd) {
    for (int idx = tid; idx < 128 * GM; idx += kThreads) {
      const int j = idx / GM, r = idx - j * GM;
      s_sq[idx] = r < group ? a.ws_sq[(row0 + r) * 128 + j] : 0.f;
    }
  }
  if (tid < 16) {
    s_kc[tid] = tid < (1 << KCB) ? a.k_centroids[tid] : 0.f;
    s_vc[tid] = tid < (1 << a.v_bits) ? a.v_centroids[tid] : 0.f;
  }
  __syncthreads();

  const int64_t t_begin = (int64_t)chunk * a.tokens_per_cta;
  const int64_t t_end = a.n_tokens < t_begin + a.tokens_per_cta ? a.n_tokens : t_begin + a.tokens_per_cta;
  const uint32_t* kbase = a.k_codes + head * a.k_head_stride;
  const uint32_t* sbase = kProd ? a.k_signs + head * a.s_head_stride : nullptr;
  const float* knb = a.k_norms + head * a.tok_head_stride;
  const float* kgb = kProd ? a.k_gammas + head * a.tok_head_stride : nullptr;
  const uint32_t* vbase = a.v_codes + head * a.v_head_stride;
  const float* vnb = a.v_norms + head * a.tok_head_stride;

  // value coordinate j = tid (j < 129): its code's place in a value row
  const int vb = a.v_bits;
  const uint32_t vmask = (1u << vb) - 1u;
  const int vo = tid * vb, vwi = vo >> 5, vsh = vo & 31;
  const bool vtwo = vsh + vb > 32;
  const bool jv = tid < kNcv;

  float m_run[RPW], l_run[RPW];
#pragma unroll
  for (int k = 0; k < RPW; ++k) {
    m_run[k] = -INFINITY;
    l_run[k] = 0.f;
  }
  float accv[GM];
#pragma unroll
  for (int r = 0; r < GM; ++r) accv[r] = 0.f;

  for (int64_t t0 = t_begin; t0 < t_end; t0 += kAttnSub) {
    const int nt = (int)((t_end - t0) < kAttnSub ? (t_end - t0) : kAttnSub);
    // ---- logits: thread tid <-> token t0 + tid
    {
      float lg[GM];
      if (tid < nt) {
        const int64_t t = t0 + tid;
        uint32_t kw[KW];
        const uint32_t* kr = kbase + t * a.ldk;
#pragma unroll
        for (int w = 0; w < KW; ++w) kw[w] = __ldg(kr + w);
        float acc[GM];
#pragma unroll
        for (int r = 0; r < GM; ++r) acc[r] = 0.f;
#pragma unroll
        for (int j = 0; j < NCK; ++j) {
          const int o = j * KCB, wi = o >> 5, sh = o & 31;
          uint32_t code = kw[wi] >> sh;
          if (sh + KCB > 32) code |= kw[wi + 1] << (32 - sh);
          code &= (1u << KCB) - 1u;
          const float c = s_kc[code];
          const float4* qv = reinterpret_cast<const float4*>(s_q + j * GM);
#pragma unroll
          for (int r4 = 0; r4 < GM / 4; ++r4) {
            const float4 qq = qv[r4];
            acc[4 * r4 + 0] = fmaf(c, qq.x, acc[4 * r4 + 0]);
            acc[4 * r4 + 1] = fmaf(c, qq.y, acc[4 * r4 + 1]);
            acc[4 * r4 + 2] = fmaf(c, qq.z, acc[4 * r4 + 2]);
            acc[4 * r4 + 3] = fmaf(c, qq.w, acc[4 * r4 + 3]);
          }
        }
        if (kProd) {
          uint32_t sw[4];
#pragma unroll
          for (int w = 0; w < 4; ++w) sw[w] = __ldg(sbase + t * a.lds + w);
          float accs[GM];
#pragma unroll
          for (int r = 0; r < GM; ++r) accs[r] = 0.f;
#pragma unroll
          for (int j = 0; j < 128; ++j) {
            const float sg = ((sw[j >> 5] >> (j & 31)) & 1u) ? 1.f : -1.f;
            const float4* sv = reinterpret_cast<const float4*>(s_sq + j * GM);
#pragma unroll
            for (int r4 = 0; r4 < GM / 4; ++r4) {
              const float4 qq = sv[r4];
              accs[4 * r4 + 0] = fmaf(sg, qq.x, accs[4 * r4 + 0]);
              accs[4 * r4 + 1] = fmaf(sg, qq.y, accs[4 * r4 + 1]);
              accs[4 * r4 + 2] = fmaf(sg, qq.z, accs[4 * r4 + 2]);
              accs[4 * r4 + 3] = fmaf(sg, qq.w, accs[4 * r4 + 3]);
            }
          }
          const float gs = __ldg(kgb + t) * a.qjl_scale;
#pragma unroll
          for (int r = 0; r < GM; ++r) acc[r] = fmaf(gs, accs[r], acc[r]);
        }
        const float kn = __ldg(knb + t) * a.scale;
#pragma unroll
        for (int r = 0; r < GM; ++r) lg[r] = kn * acc[r];
        s_vn[tid] = __ldg(vnb + t);
      } else {
#pragma unroll
        for (int r = 0; r < GM; ++r) lg[r] = 0.f;  // never read: tokens >= nt are skipped below
        s_vn[tid] = 0.f;
      }
      float4* pr = reinterpret_cast<float4*>(s_p + tid * GM);
#pragma unroll
      for (int r4 = 0; r4 < GM / 4; ++r4) pr[r4] = make_float4(lg[4 * r4], lg[4 * r4 + 1], lg[4 * r4 + 2], lg[4 * r4 + 3]);
    }
    __syncthreads();
    // ---- online softmax: warp w owns rows w, w + 8, ...
#pragma unroll
    for (int k = 0; k < RPW; ++k) {
      const int r = warp + kWarps * k;
      if (r < group) {
        float mx = -INFINITY;
        for (int t = lane; t < nt; t += 32) mx = fmaxf(mx, s_p[t * GM + r]);
        mx = warp_max(mx);
        const float m_new = fmaxf(m_run[k], mx);
        float sum = 0.f;
        for (int t = lane; t < nt; t += 32) {
          const float p = expf(s_p[t * GM + r] - m_new);
          sum += p;
          s_p[t * GM + r] = p * s_vn[t];
        }
        sum = warp_sum(sum);
        const float alpha = expf(m_run[k] - m_new);  // 0 on the first sub-chunk
        l_run[k] = fmaf(l_run[k], alpha, sum);
        m_run[k] = m_new;
        if (lane == 0) s_alpha[r] = alpha;
      } else if (lane == 0) {
        s_alpha[r] = 0.f;
      }
    }
    __syncthreads();
    // ---- value sums in the rotated domain: thread tid <-> value coordinate j
    if (jv) {
#pragma unroll
      for (int r = 0; r < GM; ++r) accv[r] *= s_alpha[r];
      const uint32_t* vr = vbase + t0 * a.ldv + vwi;
      for (int t = 0; t < nt; ++t, vr += a.ldv) {
        uint32_t code = __ldg(vr) >> vsh;
        if (vtwo) code |= __ldg(vr + 1) << (32 - vsh);
        const float c = s_vc[code & vmask];
        const float4* pp = reinterpret_cast<const float4*>(s_p + t * GM);
#pragma unroll
        for (int r4 = 0; r4 < GM / 4; ++r4) {
          const float4 p = pp[r4];
          accv[4 * r4 + 0] = fmaf(p.x, c, accv[4 * r4 + 0]);
          accv[4 * r4 + 1] = fmaf(p.y, c, accv[4 * r4 + 1]);
          accv[4 * r4 + 2] = fmaf(p.z, c, accv[4 * r4 + 2]);
          accv[4 * r4 + 3] = fmaf(p.w, c, accv[4 * r4 + 3]);
        }
      }
    }
    __syncthreads();
  }

#pragma unroll
  for (int k = 0; k < RPW; ++k) {
    const int r = warp + kWarps * k;
    if (r < group && lane == 0) {
      float* ml = a.ws_ml + ((row0 + r) * a.n_chunks + chunk) * 2;
      ml[0] = m_run[k];
      ml[1] = l_run[k];
    }
  }
  if (jv) {
#pragma unroll
    for (int r = 0; r < GM; ++r)
      if (r < group) a.ws_acc[((row0 + r) * a.n_chunks + chunk) * kAttnAS + tid] = accv[r];
  }
}

// ------------------------------------------------------------------ 3. merge + inverse sandwich
// One CTA of 256 threads per query row.
__global__ void __launch_bounds__(kThreads) attn_combine_kernel(AttnArgs a) {
  __shared__ float s_w[kAttnMaxChunks];
  __shared__ float s_y[kAttnAS];
  __shared__ float s_red[kWarps];
  const int64_t row = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nc = a.n_chunks;
  const float* ml = a.ws_ml + row * nc * 2;

  float mx = -INFINITY;
  for (int c = tid; c < nc; c += kThreads) mx = fmaxf(mx, ml[2 * c]);
  mx = warp_max(mx);
  if (lane == 0) s_red[warp] = mx;
  __syncthreads();
  float M = s_red[0];
#pragma unroll
  for (int w = 1; w < kWarps; ++w) M = fmaxf(M, s_red[w]);
  __syncthreads();

  float sum = 0.f;
  for (int c = tid; c < nc; c += kThreads) {
    const float w = ml[2 * c] == -INFINITY ? 0.f : expf(ml[2 * c] - M);  // an empty chunk weighs nothing
    s_w[c] = w;
    sum = fmaf(w, ml[2 * c + 1], sum);
  }
  sum = warp_sum(sum);
  if (lane == 0) s_red[warp] = sum;
  __syncthreads();
  float L = 0.f;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) L += s_red[w];  // >= 1: the chunk holding the largest logit adds >= 1
  const float inv = L > 0.f ? 1.f / L : 0.f;        // (0 only for a paged sequence with no tokens: output 0)

  if (tid < kNcv) {
    const float* acc = a.ws_acc + row * nc * kAttnAS + tid;
    float y = 0.f;
    for (int c = 0; c < nc; ++c) y = fmaf(s_w[c], acc[(int64_t)c * kAttnAS], y);
    s_y[tid] = y * inv;
  }
  __syncthreads();
  if (tid < kGroups) {
    const float4 r = __ldg(reinterpret_cast<const float4*>(a.v_rotors) + tid);
    float m[9];
    rotor_matrix(r.x, r.y, r.z, r.w, m);
    const float y0 = s_y[3 * tid], y1 = s_y[3 * tid + 1], y2 = s_y[3 * tid + 2];
#pragma unroll
    for (int i = 0; i < 3; ++i) {
      const int idx = 3 * tid + i;
      if (idx >= 128) break;
      const float x = fmaf(m[6 + i], y2, fmaf(m[3 + i], y1, m[i] * y0));  // M^T y
      const int64_t off = row * a.ldo + idx;
      if (a.odtype == KVRQ_F32) reinterpret_cast<float*>(a.out)[off] = x;
      else if (a.odtype == KVRQ_BF16) reinterpret_cast<__nv_bfloat16*>(a.out)[off] = __float2bfloat16_rn(x);
      else reinterpret_cast<__half*>(a.out)[off] = __float2half_rn(x);
    }
  }
}

template <int METHOD, int KCB>
static cudaError_t launch_chunks(const AttnArgs& a, cudaStream_t st) {
  const dim3 grid((unsigned)a.n_chunks, (unsigned)a.n_heads);
  if (a.group <= 8) attn_chunk_kernel<METHOD, KCB, 8><<<grid, kThreads, 0, st>>>(a);
  else attn_chunk_kernel<METHOD, KCB, 16><<<grid, kThreads, 0, st>>>(a);
  return cudaGetLastError();
}

template <int METHOD>
static cudaError_t launch_chunks_bits(int kcb, const AttnArgs& a, cudaStream_t st) {
  switch (kcb) {
    case 1: return launch_chunks<METHOD, 1>(a, st);
    case 2: return launch_chunks<METHOD, 2>(a, st);
    case 3: return launch_chunks<METHOD, 3>(a, st);
    case 4: return launch_chunks<METHOD, 4>(a, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace attn

int64_t attn_tokens_per_cta(int64_t n_heads, int64_t n_tokens) {
  const int64_t n_sub = (n_tokens + kAttnSub - 1) / kAttnSub;
  int64_t k = n_heads * n_sub / 2048;  // aim at 2,048 or more chunk CTAs
  if (k < 1) k = 1;
  if (k > 16) k = 16;
  const int64_t k_min = (n_sub + kAttnMaxChunks - 1) / kAttnMaxChunks;
  if (k < k_min) k = k_min;
  return k * kAttnSub;
}

int64_t attn_tc_tokens_per_item(int64_t n_heads, int64_t n_tokens) {
  // Every decode warpgroup of the persistent kernel takes whole items in turn: 444 workers (three
  // per SM of a 148-SM B200; a sizing rule, not a device query). A head's T tiles are cut into
  // items of k tiles (the last one shorter); the slowest worker runs ceil(items / 444) items of
  // k tiles plus about one tile's worth of set-up each, and k is chosen to make that smallest
  // (ties: fewer items, so fewer partials to merge), with at most kAttnMaxChunks items per head.
  constexpr int64_t kWorkers = 148 * kAttnTcParts;
  const int64_t T = (n_tokens + 127) / 128;
  if (T <= 1) return 128;
  int64_t best_k = T, best_cost = -1;
  for (int64_t ip = 1; ip <= T && ip <= kAttnMaxChunks; ++ip) {
    const int64_t k = (T + ip - 1) / ip;
    const int64_t items = (T + k - 1) / k;
    if (items != ip) continue;  // the same k as a smaller ip
    const int64_t cost = ((n_heads * items + kWorkers - 1) / kWorkers) * (k + 1);
    if (best_cost < 0 || cost < best_cost) {
      best_cost = cost;
      best_k = k;
    }
  }
  return best_k * 128;
}

size_t attn_workspace_bytes(int64_t n_heads, int group, int64_t n_tokens) {
  const int64_t rows = n_heads * group;
  const int64_t tpc = attn_tokens_per_cta(n_heads, n_tokens);
  const int64_t nc_cuda = (n_tokens + tpc - 1) / tpc;
  const int64_t tpi = attn_tc_tokens_per_item(n_heads, n_tokens);
  const int64_t nc_tc = (n_tokens + tpi - 1) / tpi;
  const int64_t nc = nc_cuda > nc_tc ? nc_cuda : nc_tc;
  return (size_t)rows * 4 * (kAttnQS + 128 + nc * (kAttnAS + 2));
}

cudaError_t launch_attention(int k_method, int k_cbits, AttnArgs a, cudaStream_t st, int num_sms) {
  const unsigned rows = (unsigned)(a.n_heads * a.group);
  const bool tc = attn_tc_supported(k_method, k_cbits, a.v_bits, a.group);
  if (tc) {
    a.tokens_per_cta = attn_tc_tokens_per_item(a.n_heads, a.n_tokens);
    a.n_chunks = (int)((a.n_tokens + a.tokens_per_cta - 1) / a.tokens_per_cta);
  } else {
    a.tokens_per_cta = attn_tokens_per_cta(a.n_heads, a.n_tokens);
    a.n_chunks = (int)((a.n_tokens + a.tokens_per_cta - 1) / a.tokens_per_cta);
  }
  attn::attn_rotate_q_kernel<<<rows, 128, 0, st>>>(a, k_method);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (tc) {
    e = launch_attention_tc(k_method, k_cbits, a, st, num_sms);
    if (e != cudaSuccess) return e;
    attn::attn_combine_kernel<<<rows, attn::kThreads, 0, st>>>(a);
    return cudaGetLastError();
  }
  switch (k_method) {
    case KVRQ_RQ_MSE: e = attn::launch_chunks_bits<KVRQ_RQ_MSE>(k_cbits, a, st); break;
    case KVRQ_TQ_MSE: e = attn::launch_chunks_bits<KVRQ_TQ_MSE>(k_cbits, a, st); break;
    case KVRQ_TQ_PROD:
      e = k_cbits <= 3 ? attn::launch_chunks_bits<KVRQ_TQ_PROD>(k_cbits, a, st) : cudaErrorInvalidValue;
      break;
    default: return cudaErrorInvalidValue;
  }
  if (e != cudaSuccess) return e;
  attn::attn_combine_kernel<<<rows, attn::kThreads, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace kvrq
