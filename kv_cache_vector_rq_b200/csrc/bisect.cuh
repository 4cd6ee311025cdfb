// Binary-search scalar quantizer on the FMA pipe, shared by the RotorQuant and TurboQuant
// kernels ("TurboQuant + RotorQuant", "Codebook Calibration Fix": nearest Lloyd-Max centroid of
// a rotated coordinate; ties to the lower index).
#pragma once

#include <cuda_runtime.h>

#include "kvrq_device.cuh"

namespace kvrq {

// Binary search over the positive boundaries for b = 3 and 4 (one saturating
// step per code bit instead of one per boundary). Step s_1 compares |u| with the
// middle boundary; every later step's boundary, and the centroid magnitude, are
// selected from the earlier steps (each exactly 0 or 1) by fused multiply-adds,
// fma(s, hi - lo, lo), so each selected boundary is a float of the boundary's own
// magnitude and the 0/1 argument of the linear steps carries over. The
// magnitude of count c = sum_k s_k 2^(L-k) is evaluated by one fixed FMA
// sequence on the magnitudes M_j (row-scaled, ||x|| c[H+j], in the RotorQuant
// kernel; the unit c[H+j] in the TurboQuant one); the dequantize table runs the
// same sequence with constant 0/1 steps, so both give the same bits.
template <int BITS>
struct Bisect {
  static constexpr int H = 1 << (BITS - 1);
  float t1;          // -tau_mid B
  float t2lo, t2d;   // level-2 boundary: t2lo + s1 (t2hi - t2lo)
  float q[4];        // b = 4, level 3: q0 + s1 q1 + s2 (q2 + s1 q3)
  float kb[4], kd[4];  // magnitude: base(s1, s2) + s3 delta(s1, s2)  (b = 3: kb only)

  // sc[j] = -tau_{j+1} B, j = 0 .. H-2; M[j] = ||x|| c[H + j]
  __device__ __forceinline__ void thresholds(const float* sc) {
    if constexpr (BITS == 3) {
      t1 = sc[1];
      t2lo = sc[0];
      t2d = __fsub_rn(sc[2], sc[0]);
    } else {
      t1 = sc[3];
      t2lo = sc[1];
      t2d = __fsub_rn(sc[5], sc[1]);
      q[0] = sc[0];
      q[1] = __fsub_rn(sc[4], sc[0]);
      q[2] = __fsub_rn(sc[2], sc[0]);
      q[3] = __fsub_rn(__fsub_rn(sc[6], sc[4]), q[2]);
    }
  }
  __device__ __forceinline__ void magnitudes(const float* M) {
    if constexpr (BITS == 3) {
      kb[0] = M[0];
      kb[1] = __fsub_rn(M[2], M[0]);
      kb[2] = __fsub_rn(M[1], M[0]);
      kb[3] = __fsub_rn(__fsub_rn(M[3], M[2]), kb[2]);
    } else {
      kb[0] = M[0];
      kb[1] = __fsub_rn(M[4], M[0]);
      kb[2] = __fsub_rn(M[2], M[0]);
      kb[3] = __fsub_rn(__fsub_rn(M[6], M[4]), kb[2]);
      const float d0 = __fsub_rn(M[1], M[0]), d2 = __fsub_rn(M[3], M[2]);
      const float d4 = __fsub_rn(M[5], M[4]), d6 = __fsub_rn(M[7], M[6]);
      kd[0] = d0;
      kd[1] = __fsub_rn(d4, d0);
      kd[2] = __fsub_rn(d2, d0);
      kd[3] = __fsub_rn(__fsub_rn(d6, d4), kd[2]);
    }
  }
  // 4-entry selection f(s1, s2) = k0 + s1 k1 + s2 (k2 + s1 k3), as the kernel evaluates it
  __device__ __forceinline__ static float sel(const float* k, float s1, float s2) {
    return fmaf(s2, fmaf(s1, k[3], k[2]), fmaf(s1, k[1], k[0]));
  }
  __device__ __forceinline__ static float2 sel2(const float* k, float2 s1, float2 s2) {
    const float2 hi = __ffma2_rn(s1, make_float2(k[3], k[3]), make_float2(k[2], k[2]));
    return __ffma2_rn(s2, hi, __ffma2_rn(s1, make_float2(k[1], k[1]), make_float2(k[0], k[0])));
  }
  // magnitude of count c (dequantize table)
  __device__ __forceinline__ float mag(int c) const {
    if constexpr (BITS == 3) {
      return sel(kb, (float)((c >> 1) & 1), (float)(c & 1));
    } else {
      const float s1 = (float)((c >> 2) & 1), s2 = (float)((c >> 1) & 1), s3 = (float)(c & 1);
      return fmaf(s3, sel(kd, s1, s2), sel(kb, s1, s2));
    }
  }
  // |y'| of two coordinates -> (magnitude, count + 1/2), srow = B / ||x||
  __device__ __forceinline__ void operator()(float2 a, float srow, float2& m, float2& cnt) const {
    const float2 s1 = make_float2(fma_sat(a.x, srow, t1), fma_sat(a.y, srow, t1));
    const float2 t2 = __ffma2_rn(s1, make_float2(t2d, t2d), make_float2(t2lo, t2lo));
    const float2 s2 = make_float2(fma_sat(a.x, srow, t2.x), fma_sat(a.y, srow, t2.y));
    if constexpr (BITS == 3) {
      m = sel2(kb, s1, s2);
      cnt = __fadd2_rn(__ffma2_rn(s1, make_float2(2.f, 2.f), s2), make_float2(0.5f, 0.5f));
    } else {
      const float2 t3 = sel2(q, s1, s2);
      const float2 s3 = make_float2(fma_sat(a.x, srow, t3.x), fma_sat(a.y, srow, t3.y));
      m = __ffma2_rn(s3, sel2(kd, s1, s2), sel2(kb, s1, s2));
      const float2 c2 = __ffma2_rn(s2, make_float2(2.f, 2.f), s3);
      cnt = __fadd2_rn(__ffma2_rn(s1, make_float2(4.f, 4.f), c2), make_float2(0.5f, 0.5f));
    }
  }
};

}  // namespace kvrq
