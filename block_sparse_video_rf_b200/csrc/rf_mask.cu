// Block scores and top-k mask (K2).
//
// vllm-omni "RainFusion Attention", intro: pooled 128-token key blocks are
// ranked per query block and the highest-scoring ones are attended;
// first-frame blocks stay dense.  "Configuration": sparsity is the nominal
// dropped fraction of key blocks.  lite_boost.ops.sparse_attention, rf_v2
// pipeline: block pooling -> top-k sparse mask generation.
//
// Per (b, head): s_ij = qbar_i . kbar_j in fp32 (sequential FMA over the 128
// channels).  Row i keeps the k largest scores, equal scores going to the
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
constexpr int kPad = RF_HEAD_DIM + 1;

__device__ __forceinline__ uint32_t order_key(float f) {
  const uint32_t u = __float_as_uint(f + 0.0f);   // -0 -> +0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_value(uint32_t key) {
  return __uint_as_float((key & 0x80000000u) ? (key & 0x7FFFFFFFu) : ~key);
}

template <int QC>
__global__ void __launch_bounds__(kMaskThreads) mask_kernel(const float* __restrict__ pooled_q,
                                                           const float* __restrict__ pooled_k, int nb, int ff, int k,
                                                           int words, uint32_t* __restrict__ mask,
                                                           int* __restrict__ kept, float* __restrict__ margin) {
  extern __shared__ float smem[];
  float* qs = smem;                        // [QC][129]
  float* ks = qs + QC * kPad;              // [64][129]
  uint32_t* sc = reinterpret_cast<uint32_t*>(ks + kKChunk * kPad);   // [QC][words * 32] keys
  const int row_stride = words * 32;
  const int bn = blockIdx.y;
  const int i0 = blockIdx.x * QC;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  constexpr int RPW = QC / 8;               // query rows per warp
  const float* pq = pooled_q + (size_t)bn * nb * RF_HEAD_DIM;
  const float* pk = pooled_k + (size_t)bn * nb * RF_HEAD_DIM;

  for (int idx = tid; idx < QC * RF_HEAD_DIM; idx += kMaskThreads) {
    const int r = idx >> 7, d = idx & 127;
    qs[r * kPad + d] = (i0 + r < nb) ? pq[(size_t)(i0 + r) * RF_HEAD_DIM + d] : 0.f;
  }
  for (int j0 = 0; j0 < nb; j0 += kKChunk) {
    __syncthreads();
    for (int idx = tid; idx < kKChunk * RF_HEAD_DIM; idx += kMaskThreads) {
      const int r = idx >> 7, d = idx & 127;
      ks[r * kPad + d] = (j0 + r < nb) ? pk[(size_t)(j0 + r) * RF_HEAD_DIM + d] : 0.f;
    }
    __syncthreads();
    float acc[RPW][2];
#pragma unroll
    for (int rr = 0; rr < RPW; ++rr) acc[rr][0] = acc[rr][1] = 0.f;
#pragma unroll 4
    for (int d = 0; d < RF_HEAD_DIM; ++d) {
      const float k0 = ks[lane * kPad + d], k1 = ks[(lane + 32) * kPad + d];
#pragma unroll
      for (int rr = 0; rr < RPW; ++rr) {
        const float qv = qs[(warp * RPW + rr) * kPad + d];
        acc[rr][0] = fmaf(qv, k0, acc[rr][0]);
        acc[rr][1] = fmaf(qv, k1, acc[rr][1]);
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
    if (i >= nb) break;
    const uint32_t* keys = sc + lr * row_stride;
    uint32_t* mrow = mask + ((size_t)bn * nb + i) * words;
    const size_t ri = (size_t)bn * nb + i;
    if (i < ff || k >= nb) {
      for (int w = lane; w < words; w += 32) {
        const int valid = min(32, nb - 32 * w);
        mrow[w] = valid >= 32 ? 0xFFFFFFFFu : ((1u << valid) - 1u);
      }
      if (lane == 0) {
        kept[ri] = nb;
        margin[ri] = CUDART_INF_F;
      }
      continue;
    }
    uint32_t thr = 0;     // k-th largest key (k >= 1), else unused
    int need = 0;
    float mg = CUDART_INF_F;
    if (k > 0) {
      for (int bit = 31; bit >= 0; --bit) {
        const uint32_t cand = thr | (1u << bit);
        int cnt = 0;
        for (int j = lane; j < nb; j += 32) cnt += keys[j] >= cand;
        cnt = __reduce_add_sync(0xFFFFFFFFu, cnt);
        if (cnt >= k) thr = cand;
      }
      int gt = 0, ge = 0;
      uint32_t below = 0;
      for (int j = lane; j < nb; j += 32) {
        const uint32_t u = keys[j];
        gt += u > thr;
        ge += u >= thr;
        if (u < thr && u > below) below = u;
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
    for (int w = 0; w < words; ++w) {
      const int j = 32 * w + lane;
      const uint32_t u = j < nb ? keys[j] : 0u;
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
      kept[ri] = total;
      margin[ri] = mg;
    }
  }
}

template <int QC>
size_t mask_smem_bytes(int words) {
  return sizeof(float) * (size_t)(QC * kPad + kKChunk * kPad) + sizeof(uint32_t) * (size_t)QC * words * 32;
}

template <int QC>
cudaError_t launch_mask_qc(const float* pq, const float* pk, int BN, int nb, int ff, int k, int words, uint32_t* mask,
                           int* kept, float* margin, cudaStream_t stream) {
  const size_t smem = mask_smem_bytes<QC>(words);
  cudaError_t e = cudaFuncSetAttribute(mask_kernel<QC>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((nb + QC - 1) / QC, BN);
  mask_kernel<QC><<<grid, kMaskThreads, smem, stream>>>(pq, pk, nb, ff, k, words, mask, kept, margin);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_mask(const float* pooled_q, const float* pooled_k, int BN, const rf_plan_t& g, uint32_t* mask,
                        int* kept, float* margin, cudaStream_t stream) {
  if (g.nb == 0) return cudaSuccess;
  const size_t limit = 200 * 1024;
  if (mask_smem_bytes<32>(g.mask_words) <= limit)
    return launch_mask_qc<32>(pooled_q, pooled_k, BN, g.nb, g.ff, g.k, g.mask_words, mask, kept, margin, stream);
  if (mask_smem_bytes<16>(g.mask_words) <= limit)
    return launch_mask_qc<16>(pooled_q, pooled_k, BN, g.nb, g.ff, g.k, g.mask_words, mask, kept, margin, stream);
  return launch_mask_qc<8>(pooled_q, pooled_k, BN, g.nb, g.ff, g.k, g.mask_words, mask, kept, margin, stream);
}

}  // namespace rf
