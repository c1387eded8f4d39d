// Element types of the caller's q, k, v and out: bf16 or fp16 (both 16-bit;
// the reorder copies their bits unchanged, only the fp32 pooling and the
// attention's operand and output formats depend on which).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

namespace rf {

// Adds the 8 16-bit values of `u` (low half of each word first) to acc, as fp32.
template <bool kF16>
__device__ __forceinline__ void acc_half8(float (&acc)[8], const uint4& u) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    if (kF16) {
      const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w[i]));
      acc[2 * i] += f.x;
      acc[2 * i + 1] += f.y;
    } else {
      acc[2 * i] += __uint_as_float(w[i] << 16);
      acc[2 * i + 1] += __uint_as_float(w[i] & 0xFFFF0000u);
    }
  }
}

// The 8 16-bit values of `u` (low half of each word first) as fp32.
template <bool kF16>
__device__ __forceinline__ void unpack_half8(const uint4& u, float (&f)[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    if (kF16) {
      const float2 h = __half22float2(*reinterpret_cast<const __half2*>(&w[i]));
      f[2 * i] = h.x;
      f[2 * i + 1] = h.y;
    } else {
      f[2 * i] = __uint_as_float(w[i] << 16);
      f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
  }
}

// lo += low half of w, hi += high half, each 16-bit value widened exactly to
// fp32 and the sum rounded to nearest (the sm_100 mixed-precision add, one
// instruction per value instead of an unpack and an add).
template <bool kF16>
__device__ __forceinline__ void add_half2_to(uint32_t w, float& lo, float& hi) {
  if (kF16)
    asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %2;\n\tadd.rn.f32.f16 %0, l, %0;\n\tadd.rn.f32.f16 %1, h, %1;\n\t}"
        : "+f"(lo), "+f"(hi)
        : "r"(w));
  else
    asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %2;\n\tadd.rn.f32.bf16 %0, l, %0;\n\tadd.rn.f32.bf16 %1, h, %1;\n\t}"
        : "+f"(lo), "+f"(hi)
        : "r"(w));
}

}  // namespace rf
