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

// The two 16-bit values of one word (low half first) as fp32.
template <bool kF16>
__device__ __forceinline__ void unpack_half2(uint32_t w, float& lo, float& hi) {
  if (kF16) {
    const float2 h = __half22float2(*reinterpret_cast<const __half2*>(&w));
    lo = h.x;
    hi = h.y;
  } else {
    lo = __uint_as_float(w << 16);
    hi = __uint_as_float(w & 0xFFFF0000u);
  }
}

}  // namespace rf
