// Device-side building blocks for sm_100a: mbarriers, TMA tensor and bulk
// copies, proxy fences, the bounded-wait status word, and dtype traits.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

namespace kvrq {

// Kernels get the address of a device status word; a bounded wait that runs
// out sets bit 0, an inconsistent launch sets bit 1. The host reads and
// clears it (kvrq_device_status).
constexpr unsigned kStatusTimeout = 1u;
constexpr unsigned kStatusBadLaunch = 2u;

// Upper bound on mbarrier polls before a wait gives up (each try_wait may
// itself suspend for a bounded time): well above any legitimate wait.
constexpr uint32_t kSpinLimit = 1u << 24;

__device__ __forceinline__ void record_status(unsigned* status, unsigned bits) {
  if (status) atomicOr(status, bits);
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ------------------------------------------------------------------ mbarrier
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

// Makes barrier initialisation visible to the async (TMA) proxy.
__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t phase) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(phase)
      : "memory");
  return ok != 0;
}

// Bounded wait for the phase with parity `phase` to complete. Returns false
// (and records a time-out) if it did not complete within kSpinLimit polls.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t phase, unsigned* status) {
  for (uint32_t i = 0; i < kSpinLimit; ++i)
    if (mbar_try_wait(bar, phase)) return true;
  record_status(status, kStatusTimeout);
  return false;
}

// ------------------------------------------------------------------ TMA / bulk copies
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// 2D tiled load of box (c0 = inner coordinate, c1 = row) into shared memory,
// completing `bytes` of transaction count on `bar`.
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int32_t c0, int32_t c1,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(smem_u32(bar))
      : "memory");
}

// 2D tiled store of a shared-memory box; out-of-range rows are not written.
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, int32_t c0, int32_t c1, const void* src) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.tile.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(c0), "r"(c1), "r"(smem_u32(src))
               : "memory");
}

// Contiguous global -> shared copy (addresses 16-byte aligned, bytes % 16 == 0).
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// Contiguous shared -> global copy (same alignment rules), in a bulk group.
__device__ __forceinline__ void bulk_store(void* dst, const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(reinterpret_cast<uint64_t>(dst)),
               "r"(smem_u32(src)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }

// Wait until at most N committed bulk groups still read shared memory.
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}

// Wait until at most N committed bulk groups are still in flight.
template <int N>
__device__ __forceinline__ void bulk_wait_all() {
  asm volatile("cp.async.bulk.wait_group %0;" ::"n"(N) : "memory");
}

// ------------------------------------------------------------------ dtypes
// Element traits for the three vector dtypes. A 16-byte chunk holds
// kPerChunk elements; `unpack` turns a chunk into floats, `pack` back.
template <typename T>
struct Elem;

template <>
struct Elem<float> {
  static constexpr int kPerChunk = 4;
  __device__ __forceinline__ static void unpack(const uint4& c, float* f) {
    f[0] = __uint_as_float(c.x);
    f[1] = __uint_as_float(c.y);
    f[2] = __uint_as_float(c.z);
    f[3] = __uint_as_float(c.w);
  }
  __device__ __forceinline__ static uint4 pack(const float* f) {
    return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]), __float_as_uint(f[3]));
  }
  __device__ __forceinline__ static float to_float(float v) { return v; }
  __device__ __forceinline__ static float from_float(float v) { return v; }
};

template <>
struct Elem<__half> {
  static constexpr int kPerChunk = 8;
  __device__ __forceinline__ static float2 h2f(uint32_t w) {
    __half2 h = *reinterpret_cast<__half2*>(&w);
    return __half22float2(h);
  }
  __device__ __forceinline__ static uint32_t f2h(float a, float b) {
    __half2 h = __floats2half2_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
  }
  __device__ __forceinline__ static void unpack(const uint4& c, float* f) {
    float2 t;
    t = h2f(c.x); f[0] = t.x; f[1] = t.y;
    t = h2f(c.y); f[2] = t.x; f[3] = t.y;
    t = h2f(c.z); f[4] = t.x; f[5] = t.y;
    t = h2f(c.w); f[6] = t.x; f[7] = t.y;
  }
  __device__ __forceinline__ static uint4 pack(const float* f) {
    return make_uint4(f2h(f[0], f[1]), f2h(f[2], f[3]), f2h(f[4], f[5]), f2h(f[6], f[7]));
  }
  __device__ __forceinline__ static float to_float(__half v) { return __half2float(v); }
  __device__ __forceinline__ static __half from_float(float v) { return __float2half_rn(v); }
};

template <>
struct Elem<__nv_bfloat16> {
  static constexpr int kPerChunk = 8;
  __device__ __forceinline__ static float2 h2f(uint32_t w) {
    __nv_bfloat162 h = *reinterpret_cast<__nv_bfloat162*>(&w);
    return __bfloat1622float2(h);
  }
  __device__ __forceinline__ static uint32_t f2h(float a, float b) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
  }
  __device__ __forceinline__ static void unpack(const uint4& c, float* f) {
    float2 t;
    t = h2f(c.x); f[0] = t.x; f[1] = t.y;
    t = h2f(c.y); f[2] = t.x; f[3] = t.y;
    t = h2f(c.z); f[4] = t.x; f[5] = t.y;
    t = h2f(c.w); f[6] = t.x; f[7] = t.y;
  }
  __device__ __forceinline__ static uint4 pack(const float* f) {
    return make_uint4(f2h(f[0], f[1]), f2h(f[2], f[3]), f2h(f[4], f[5]), f2h(f[6], f[7]));
  }
  __device__ __forceinline__ static float to_float(__nv_bfloat16 v) { return __bfloat162float(v); }
  __device__ __forceinline__ static __nv_bfloat16 from_float(float v) { return __float2bfloat16_rn(v); }
};

// ------------------------------------------------------------------ rotor matrix
// The sandwich v -> R v R~ of the Cl(3,0) rotor R = s + b12 e12 + b13 e13 + b23 e23
// is linear in v; its matrix is that of the quaternion q = (w, x, y, z) =
// (s, -b23, b13, -b12) acting by q v q*, written in the homogeneous form (exact
// for any R, unit or not). Row-major m[0..8]. The inverse sandwich R~ v R has
// the transposed matrix.
__device__ __forceinline__ void rotor_matrix(float s, float b12, float b13, float b23, float* m) {
  const float w = s, x = -b23, y = b13, z = -b12;
  const float ww = w * w, xx = x * x, yy = y * y, zz = z * z;
  m[0] = ww + xx - yy - zz;
  m[1] = 2.f * (x * y - w * z);
  m[2] = 2.f * (x * z + w * y);
  m[3] = 2.f * (x * y + w * z);
  m[4] = ww - xx + yy - zz;
  m[5] = 2.f * (y * z - w * x);
  m[6] = 2.f * (x * z - w * y);
  m[7] = 2.f * (y * z + w * x);
  m[8] = ww - xx - yy + zz;
}

}  // namespace kvrq
