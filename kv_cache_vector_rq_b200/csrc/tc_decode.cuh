// Shared pieces of the kernels that decode packed codes into fp16 tensor-core
// operands: the replicated decode tables, bit-field extraction from a code row
// held in registers, and a warpgroup-wide vote.
#pragma once

#include <stdint.h>

#include "kvrq_device.cuh"

namespace kvrq {

// Decode table of the stored codes (width b): an f-bit field of P codes maps to
// P fp16 centroids (EW 32-bit words); every entry is replicated R times, R
// consecutive copies filling 128 bytes, and lane l reads copy l % R, so the
// lanes of one shared-memory wavefront (8, 16 or 32 lanes for 16-, 8- and
// 4-byte entries) hit distinct banks whatever the field values.
template <int BITS>
struct Dec {
  static constexpr int FB = BITS == 3 ? 6 : 8;  // field bits
  static constexpr int P = FB / BITS;            // codes per field: 8, 4, 2, 2
  static constexpr int EW = P / 2;               // words per entry
  static constexpr int EB = 4 * EW;
  static constexpr int R = 128 / EB;             // replicas
  static constexpr int ENT = 1 << FB;
  static constexpr int BYTES = ENT * 128;
};

// Barrier `id` among the 128 threads of a warpgroup; returns the AND of `pred` over them.
__device__ __forceinline__ bool wg_all(bool pred, int id) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, %2, 128, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(pred ? 1u : 0u), "r"(id)
      : "memory");
  return r != 0;
}

// Barrier `id` among the 128 threads of a warpgroup; returns the OR of `pred` over them.
__device__ __forceinline__ bool wg_any(bool pred, int id) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, 128, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(pred ? 1u : 0u), "r"(id)
      : "memory");
  return r != 0;
}

// field of `FB` bits starting at bit `bit` of the little-endian stream in w[0..NW)
template <int FB, int NW>
__device__ __forceinline__ uint32_t field(const uint32_t (&w)[NW], int bit) {
  const int wi = bit >> 5, sh = bit & 31;
  uint32_t v = w[wi] >> sh;
  if (sh + FB > 32 && wi + 1 < NW) v |= w[wi + 1] << (32 - sh);
  return v & ((1u << FB) - 1u);
}

}  // namespace kvrq
