// Block scores and top-k mask (K2).
//
// vllm-omni "RainFusion Attention", intro: pooled 128-token key blocks are
// ranked per query block and the highest-scoring ones are attended;
// first-frame blocks stay dense.  "Configuration": sparsity is the nominal
// dropped fraction of key blocks.  lite_boost.ops.sparse_attention, rf_v2
// pipeline: block pooling -> top-k sparse mask generation.
//
// Per (b, head): s_ij = qbar_i . kbar_j in fp32 (sequential FMA over the 128
// channels), i over the query geometry's blocks, j over the key geometry's
// (the same unless k and v have their own, lite_boost latent_shape_k).  Row i keeps the k largest scores, equal scores going to the
// lower block index, plus the first-frame blocks; first-frame rows keep
// everything.  The k-th score is found by a 32-step MSB-first search over
// order-preserving integer keys, one warp per row.
#include <cuda_runtime.h>
#include <math_constants.h>

#include "rf_kernels.h"

namespace rf {

namespace {

constexpr int kMaskThreads = 256;
constexpr int kKChunk = 64;
constexpr int kPad = RF_HEAD_DIM + 4;   // row stride in floats: 16-byte aligned, float4 loads conflict-free

__device__ __forceinline__ uint32_t order_key(float f) {
  const uint32_t u = __float_as_uint(f + 0.0f);   // -0 -> +0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_value(uint32_t key) {
  return __uint_as_float((key & 0x80000000u) ? (key & 0x7FFFFFFFu) : ~key);
}

// Loads rows [r0, r0 + 64) of a pooled tensor ([nb, 128] fp32) as float4s
// into registers (8 per thread); rows past nb read as zero.
__device__ __forceinline__ void load_chunk(const float* __restrict__ src, int r0, int nb, float4 (&reg)[8]) {
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int idx = threadIdx.x + i * kMaskThreads;   // float4 index within the chunk
    const int r = idx >> 5, d4 = idx & 31;
    reg[i] = (r0 + r < nb) ? __ldg(reinterpret_cast<const float4*>(src + (size_t)(r0 + r) * RF_HEAD_DIM) + d4)
                           : make_float4(0.f, 0.f, 0.f, 0.f);
  }
}
__device__ __forceinline__ void store_chunk(float* dst, const float4 (&reg)[8]) {
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int idx = threadIdx.x + i * kMaskThreads;
    const int r = idx >> 5, d4 = idx & 31;
    *reinterpret_cast<float4*>(dst + r * kPad + 4 * d4) = reg[i];
  }
}

// Top-k selection of one score row by one warp.  Lane l holds the keys of
// blocks l, l + 32, ..., in registers (PL per lane: nb <= 32 PL); padding
// keys are 0, below every real key.  The k-th largest key is built bit by bit
// (MSB first); blocks above it are kept, and of the blocks equal to it the
// lowest indices fill the remaining places.  First-frame blocks are always
// kept; first-frame rows (and k >= nb) keep every block.
template <int PL>
__device__ __forceinline__ void select_row(const uint32_t* __restrict__ keys_s, int nb, int ff, int k, int words,
                                           bool dense_row, uint32_t* __restrict__ mrow, int* __restrict__ kept_out,
                                           float* __restrict__ margin_out) {
  const int lane = threadIdx.x & 31;
  if (dense_row || k >= nb) {
    for (int w = lane; w < words; w += 32) {
      const int valid = min(32, nb - 32 * w);
      mrow[w] = valid >= 32 ? 0xFFFFFFFFu : ((1u << valid) - 1u);
    }
    if (lane == 0) {
      *kept_out = nb;
      *margin_out = CUDART_INF_F;
    }
    return;
  }
  uint32_t key[PL];
#pragma unroll
  for (int w = 0; w < PL; ++w) {
    const int j = 32 * w + lane;
    key[w] = (w < words && j < nb) ? keys_s[j] : 0u;
  }
  uint32_t thr = 0;
  int need = 0;
  float mg = CUDART_INF_F;
  if (k > 0) {
#pragma unroll 1
    for (int bit = 31; bit >= 0; --bit) {
      const uint32_t cand = thr | (1u << bit);
      int cnt = 0;
#pragma unroll
      for (int w = 0; w < PL; ++w) cnt += key[w] >= cand;
      if (__reduce_add_sync(0xFFFFFFFFu, cnt) >= k) thr = cand;
    }
    int gt = 0, ge = 0;
    uint32_t below = 0;
#pragma unroll
    for (int w = 0; w < PL; ++w) {
      const uint32_t u = key[w];
      gt += u > thr;
      ge += u >= thr;
      below = (u < thr && u > below) ? u : below;
    }
    gt = __reduce_add_sync(0xFFFFFFFFu, gt);
    ge = __reduce_add_sync(0xFFFFFFFFu, ge);
    below = __reduce_max_sync(0xFFFFFFFFu, below);
    need = k - gt;
    const float sk = key_value(thr);
    const float sk1 = (ge > k) ? sk : key_value(below);
    mg = (sk - sk1) / fmaxf(fabsf(sk), 1e-30f);
  }
  int taken = 0, total = 0;
#pragma unroll
  for (int w = 0; w < PL; ++w) {
    if (w >= words) break;
    const int j = 32 * w + lane;
    const uint32_t u = key[w];
    const bool eq = (k > 0) && j < nb && u == thr;
    const uint32_t eqm = __ballot_sync(0xFFFFFFFFu, eq);
    const int rank = __popc(eqm & ((1u << lane) - 1u));
    const bool sel = (j < nb) && ((k > 0 && u > thr) || (eq && taken + rank < need) || j < ff);
    const uint32_t bits = __ballot_sync(0xFFFFFFFFu, sel);
    taken += __popc(eqm);
    total += __popc(bits);
    if (lane == 0) mrow[w] = bits;
  }
  if (lane == 0) {
    *kept_out = total;
    *margin_out = mg;
  }
}

// nbq query blocks (the first ffq of them dense rows) against nb key blocks
// (the first ff of them forced columns); k kept per row.
template <int QC, int PL>
__global__ void __launch_bounds__(kMaskThreads) mask_kernel(const float* __restrict__ pooled_q,
                                                           const float* __restrict__ pooled_k, int nbq, int ffq,
                                                           int nb, int ff, int k, int words,
                                                           uint32_t* __restrict__ mask, int* __restrict__ kept,
                                                           float* __restrict__ margin) {
  extern __shared__ __align__(16) float smem[];
  float* qs = smem;                        // [QC][kPad]
  float* ks = qs + QC * kPad;              // [64][kPad]
  uint32_t* sc = reinterpret_cast<uint32_t*>(ks + kKChunk * kPad);   // [QC][words * 32] keys
  const int row_stride = words * 32;
  const int bn = blockIdx.y;
  const int i0 = blockIdx.x * QC;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  constexpr int RPW = QC / 8;               // query rows per warp
  const float* pq = pooled_q + (size_t)bn * nbq * RF_HEAD_DIM;
  const float* pk = pooled_k + (size_t)bn * nb * RF_HEAD_DIM;

  for (int idx = tid; idx < QC * 32; idx += kMaskThreads) {
    const int r = idx >> 5, d4 = idx & 31;
    const float4 v = (i0 + r < nbq) ? __ldg(reinterpret_cast<const float4*>(pq + (size_t)(i0 + r) * RF_HEAD_DIM) + d4)
                                   : make_float4(0.f, 0.f, 0.f, 0.f);
    *reinterpret_cast<float4*>(qs + r * kPad + 4 * d4) = v;
  }
  float4 next[8];
  load_chunk(pk, 0, nb, next);
  for (int j0 = 0; j0 < nb; j0 += kKChunk) {
    __syncthreads();                        // previous chunk consumed
    store_chunk(ks, next);
    __syncthreads();
    if (j0 + kKChunk < nb) load_chunk(pk, j0 + kKChunk, nb, next);   // in flight during the dot products
    // s_ij: each thread takes RPW query rows x key columns lane and lane + 32,
    // summing over d in order 0..127 (fp32 FMA chain per output).
    float acc[RPW][2];
#pragma unroll
    for (int rr = 0; rr < RPW; ++rr) acc[rr][0] = acc[rr][1] = 0.f;
#pragma unroll 4
    for (int d = 0; d < RF_HEAD_DIM; d += 4) {
      const float4 k0 = *reinterpret_cast<const float4*>(ks + lane * kPad + d);
      const float4 k1 = *reinterpret_cast<const float4*>(ks + (lane + 32) * kPad + d);
#pragma unroll
      for (int rr = 0; rr < RPW; ++rr) {
        const float4 qv = *reinterpret_cast<const float4*>(qs + (warp * RPW + rr) * kPad + d);
        acc[rr][0] = fmaf(qv.x, k0.x, acc[rr][0]);
        acc[rr][0] = fmaf(qv.y, k0.y, acc[rr][0]);
        acc[rr][0] = fmaf(qv.z, k0.z, acc[rr][0]);
        acc[rr][0] = fmaf(qv.w, k0.w, acc[rr][0]);
        acc[rr][1] = fmaf(qv.x, k1.x, acc[rr][1]);
        acc[rr][1] = fmaf(qv.y, k1.y, acc[rr][1]);
        acc[rr][1] = fmaf(qv.z, k1.z, acc[rr][1]);
        acc[rr][1] = fmaf(qv.w, k1.w, acc[rr][1]);
      }
    }
#pragma unroll
    for (int rr = 0; rr < RPW; ++rr) {
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        const int j = j0 + lane + 32 * c;
        if (j < row_stride) sc[(warp * RPW + rr) * row_stride + j] = (j < nb) ? order_key(acc[rr][c]) : 0u;
      }
    }
  }
  __syncthreads();
  for (int rr = 0; rr < RPW; ++rr) {
    const int lr = warp * RPW + rr;
    const int i = i0 + lr;
    if (i >= nbq) break;
    select_row<PL>(sc + lr * row_stride, nb, ff, k, words, i < ffq, mask + ((size_t)bn * nbq + i) * words,
                   kept + (size_t)bn * nbq + i, margin + (size_t)bn * nbq + i);
  }
}

template <int QC>
size_t mask_smem_bytes(int words) {
  return sizeof(float) * (size_t)(QC * kPad + kKChunk * kPad) + sizeof(uint32_t) * (size_t)QC * words * 32;
}

template <int QC, int PL>
cudaError_t launch_mask_qc_pl(const float* pq, const float* pk, int BN, const rf_plan_t& g, const rf_plan_t& gk,
                              uint32_t* mask, int* kept, float* margin, cudaStream_t stream) {
  const size_t smem = mask_smem_bytes<QC>(gk.mask_words);
  cudaError_t e = cudaFuncSetAttribute(mask_kernel<QC, PL>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((g.nb + QC - 1) / QC, BN);
  mask_kernel<QC, PL><<<grid, kMaskThreads, smem, stream>>>(pq, pk, g.nb, g.ff, gk.nb, gk.ff, gk.k, gk.mask_words,
                                                            mask, kept, margin);
  return cudaGetLastError();
}

template <int QC>
cudaError_t launch_mask_qc(const float* pq, const float* pk, int BN, const rf_plan_t& g, const rf_plan_t& gk,
                           uint32_t* mask, int* kept, float* margin, cudaStream_t stream) {
  const int words = gk.mask_words;
  if (words <= 16) return launch_mask_qc_pl<QC, 16>(pq, pk, BN, g, gk, mask, kept, margin, stream);
  if (words <= 32) return launch_mask_qc_pl<QC, 32>(pq, pk, BN, g, gk, mask, kept, margin, stream);
  return launch_mask_qc_pl<QC, 128>(pq, pk, BN, g, gk, mask, kept, margin, stream);
}

}  // namespace

cudaError_t launch_mask(const float* pooled_q, const float* pooled_k, int BN, const rf_plan_t& g,
                        const rf_plan_t& gk, uint32_t* mask, int* kept, float* margin, cudaStream_t stream) {
  if (g.nb == 0 || gk.nb == 0) return cudaSuccess;
  const size_t limit = 200 * 1024;
  if (mask_smem_bytes<32>(gk.mask_words) <= limit)
    return launch_mask_qc<32>(pooled_q, pooled_k, BN, g, gk, mask, kept, margin, stream);
  if (mask_smem_bytes<16>(gk.mask_words) <= limit)
    return launch_mask_qc<16>(pooled_q, pooled_k, BN, g, gk, mask, kept, margin, stream);
  return launch_mask_qc<8>(pooled_q, pooled_k, BN, g, gk, mask, kept, margin, stream);
}

}  // namespace rf
