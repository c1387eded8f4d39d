// fp8 e4m3 quantisation of the reordered q, k, v (the fp8 precision of the
// attention).
//
// lite_boost.ops.sparse_attention documents an fp8 precision for its
// attention; the pages fix no scaling rule.  The reading taken here: one
// fp32 scale per 128-row block of the internal layout, per tensor and head
// (the attention's own tile), scale = amax(|x|) / 448 with 448 the largest
// finite e4m3 value, code = e4m3 round-to-nearest-even, saturating, of
// x * (448 / amax) in fp32; an all-zero block has scale 0 and codes 0.  V's
// blocks are stored transposed (channel-major) so that the P V product reads
// them K-major.  vmax[head] = the largest V block scale of the head.  q is
// blocked by the query geometry, k and v by theirs.
#include <cuda_runtime.h>

#include "rf_dtype.h"
#include "rf_kernels.h"
#include "sm100_ptx.cuh"

namespace rf {

namespace {

constexpr int kQThreads = 256;                 // 16 chunks of 8 channels x 16 rows per pass
constexpr int kRowsPerPass = kQThreads / 16;
constexpr int kPasses = RF_BLOCK / kRowsPerPass;
constexpr int kVtStride = RF_BLOCK + 4;        // bytes per transposed row in shared memory

// Up to three tensors of one geometry (S_int internal rows per head).
struct QuantArgs {
  const uint16_t* src[3];
  uint8_t* dst[3];
  float* scales[3];   // [BN, S_int / 128] block scales of each tensor
  int count;          // tensors in use
  int v_index;        // the tensor stored transposed, whose largest block scale goes to vmax (-1: none)
};

// One CTA = one 128-row block of one head, for each tensor in turn.
template <bool kF16>
__global__ void __launch_bounds__(kQThreads) quantize_kernel(QuantArgs a, int S_int, float* __restrict__ vmax) {
  __shared__ float red[kQThreads / 32];
  __shared__ __align__(16) uint8_t vt[RF_HEAD_DIM][kVtStride];
  const int tile = blockIdx.x, bn = blockIdx.y;
  const int n_tiles = S_int / RF_BLOCK;
  const int chunk = threadIdx.x & 15, rsub = threadIdx.x >> 4;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t base = ((int64_t)bn * S_int + (int64_t)tile * RF_BLOCK) * RF_HEAD_DIM;   // element offset
#pragma unroll 1
  for (int t = 0; t < a.count; ++t) {
    const bool transposed = t == a.v_index;
    float f[kPasses][8];
    float amax = 0.f;
#pragma unroll
    for (int p = 0; p < kPasses; ++p) {
      const uint4 u = __ldcs(reinterpret_cast<const uint4*>(a.src[t] + base +
                                                            (int64_t)(p * kRowsPerPass + rsub) * RF_HEAD_DIM +
                                                            chunk * 8));
      unpack_half8<kF16>(u, f[p]);
#pragma unroll
      for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(f[p][i]));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
    if (lane == 0) red[warp] = amax;
    __syncthreads();
    amax = red[0];
#pragma unroll
    for (int i = 1; i < kQThreads / 32; ++i) amax = fmaxf(amax, red[i]);
    __syncthreads();   // red is rewritten by the next tensor
    const float inv = amax > 0.f ? __fdiv_rn(448.f, amax) : 0.f;
    const float scale = __fdiv_rn(amax, 448.f);
#pragma unroll
    for (int p = 0; p < kPasses; ++p) {
      const int r = p * kRowsPerPass + rsub;
      const uint32_t lo = pack_e4m3x4(__fmul_rn(f[p][0], inv), __fmul_rn(f[p][1], inv), __fmul_rn(f[p][2], inv),
                                      __fmul_rn(f[p][3], inv));
      const uint32_t hi = pack_e4m3x4(__fmul_rn(f[p][4], inv), __fmul_rn(f[p][5], inv), __fmul_rn(f[p][6], inv),
                                      __fmul_rn(f[p][7], inv));
      if (!transposed) {
        *reinterpret_cast<uint2*>(a.dst[t] + base + (int64_t)r * RF_HEAD_DIM + chunk * 8) = make_uint2(lo, hi);
      } else {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          vt[chunk * 8 + i][r] = (uint8_t)(lo >> (8 * i));
          vt[chunk * 8 + 4 + i][r] = (uint8_t)(hi >> (8 * i));
        }
      }
    }
    if (threadIdx.x == 0) {
      a.scales[t][(int64_t)bn * n_tiles + tile] = scale;
      // non-negative floats order like their bit patterns
      if (transposed) atomicMax(reinterpret_cast<int*>(vmax) + bn, __float_as_int(scale));
    }
  }
  if (a.v_index < 0) return;
  __syncthreads();
  // transposed V block: 128 channel rows of 128 bytes, one word per thread and step
#pragma unroll
  for (int i = 0; i < RF_HEAD_DIM * RF_BLOCK / 4 / kQThreads; ++i) {
    const int idx = threadIdx.x + i * kQThreads;
    const int row = idx >> 5, word = idx & 31;
    const uint32_t w = *reinterpret_cast<const uint32_t*>(&vt[row][word * 4]);
    *reinterpret_cast<uint32_t*>(a.dst[a.v_index] + base + (int64_t)row * RF_BLOCK + word * 4) = w;
  }
}

}  // namespace

cudaError_t launch_quantize_fp8(const void* q_int, const void* k_int, const void* v_int, int dtype, int BN,
                                const rf_plan_t& g, const rf_plan_t& gk, uint8_t* q8, uint8_t* k8, uint8_t* v8,
                                float* scales, float* vmax, cudaStream_t stream) {
  cudaError_t e = cudaMemsetAsync(vmax, 0, sizeof(float) * BN, stream);
  if (e != cudaSuccess) return e;
  auto kern = dtype == RF_F16 ? quantize_kernel<true> : quantize_kernel<false>;
  auto s16 = [](const void* x) { return static_cast<const uint16_t*>(x); };
  float* sq = scales;
  float* sk = sq + (size_t)BN * g.n_tiles;
  float* sv = sk + (size_t)BN * gk.n_tiles;
  if (g.S_int == gk.S_int) {   // one internal length: one pass over q, k, v
    QuantArgs a{{s16(q_int), s16(k_int), s16(v_int)}, {q8, k8, v8}, {sq, sk, sv}, 3, 2};
    kern<<<dim3(g.n_tiles, BN), kQThreads, 0, stream>>>(a, g.S_int, vmax);
    return cudaGetLastError();
  }
  QuantArgs a{{s16(q_int), nullptr, nullptr}, {q8, nullptr, nullptr}, {sq, nullptr, nullptr}, 1, -1};
  kern<<<dim3(g.n_tiles, BN), kQThreads, 0, stream>>>(a, g.S_int, vmax);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  a = QuantArgs{{s16(k_int), s16(v_int), nullptr}, {k8, v8, nullptr}, {sk, sv, nullptr}, 2, 1};
  kern<<<dim3(gk.n_tiles, BN), kQThreads, 0, stream>>>(a, gk.S_int, vmax);
  return cudaGetLastError();
}

}  // namespace rf
