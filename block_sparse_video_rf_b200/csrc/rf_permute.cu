// Token reorder with block pooling fused in (K1), and the inverse reorder
// (K4).  Both are HBM-bound row gathers/scatters of 256-byte rows.
//
// lite_boost.ops.sparse_attention, rf_v2 pipeline: token reorder, then block
// pooling; inverse reorder at the end.  vllm-omni "RainFusion Attention":
// 128-token key blocks are pooled (intro); the reorder groups video tokens
// into 8x8 tiles and promotes the non-aligned rest ("Geometry handling").
#include <cuda_runtime.h>

#include <cstring>

#include "rf_dtype.h"
#include "rf_geometry.h"
#include "rf_kernels.h"

namespace rf {

namespace {

constexpr int kPermThreads = 256;   // 16 rows x 16 chunks of 16 bytes per pass
constexpr int kRowsPerPass = kPermThreads / 16;
constexpr int kPasses = RF_BLOCK / kRowsPerPass;

// Up to three tensors of one geometry (plan g, S rows in the caller's layout).
struct PermArgs {
  const uint16_t* src[3];
  uint16_t* dst[3];
  float* pooled[2];   // block means of tensors 0 and 1 (nullptr: not pooled)
  int count;          // tensors in use
};

// One CTA = one 128-row internal tile of one (b, head), for each tensor.
// Sparse tiles also write the fp32 block means of the pooled tensors.  The
// column sums run in a fixed order (per thread over its 8 rows, then over the
// 16 row groups), so results are deterministic.  Rows are 16-bit values
// (bf16, or fp16 when kF16) copied bit for bit; only the pooling reads them as
// numbers.
template <bool kF16>
__global__ void __launch_bounds__(kPermThreads) permute_pool_kernel(PermArgs a, int layout, int B, int S, int N,
                                                                    rf_plan_t g) {
  __shared__ float red[2][kRowsPerPass][RF_HEAD_DIM];
  const int tile = blockIdx.x;
  const int bn = blockIdx.y;
  const int b = bn / N, n = bn - b * N;
  const int chunk = threadIdx.x & 15;     // 16-byte column chunk
  const int rsub = threadIdx.x >> 4;      // row within the pass
  const bool sparse = (tile * RF_BLOCK >= g.P_pad) && !g.dense;

  int64_t src_off[kPasses];
#pragma unroll
  for (int p = 0; p < kPasses; ++p) {
    const int r = tile * RF_BLOCK + p * kRowsPerPass + rsub;
    const int s = rf_src_of_row(g, r);
    src_off[p] = s < 0 ? -1 : rf_token_offset(layout, B, S, N, b, n, s) + chunk * 8;
  }
  const int64_t dst_base = ((int64_t)bn * g.S_int + (int64_t)tile * RF_BLOCK) * RF_HEAD_DIM + chunk * 8;

#pragma unroll
  for (int t = 0; t < 3; ++t) {
    if (t >= a.count) break;
    const uint16_t* src = a.src[t];
    uint16_t* dst = a.dst[t];
    uint4 buf[kPasses];
#pragma unroll
    for (int p = 0; p < kPasses; ++p) {
      buf[p] = src_off[p] < 0 ? make_uint4(0, 0, 0, 0) : __ldcs(reinterpret_cast<const uint4*>(src + src_off[p]));
    }
#pragma unroll
    for (int p = 0; p < kPasses; ++p) {
      *reinterpret_cast<uint4*>(dst + dst_base + (int64_t)(p * kRowsPerPass + rsub) * RF_HEAD_DIM) = buf[p];
    }
    if (t < 2 && sparse && a.pooled[t]) {
      float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int p = 0; p < kPasses; ++p) acc_half8<kF16>(acc, buf[p]);
#pragma unroll
      for (int i = 0; i < 8; ++i) red[t][rsub][chunk * 8 + i] = acc[i];
    }
  }
  if (!sparse) return;
  __syncthreads();
  // 256 threads: 2 tensors x 128 columns.
  const int t = threadIdx.x >> 7, c = threadIdx.x & 127;
  if (!a.pooled[t]) return;
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < kRowsPerPass; ++i) s += red[t][i][c];
  const int blk = tile - g.P_pad / RF_BLOCK;
  a.pooled[t][((int64_t)bn * g.nb + blk) * RF_HEAD_DIM + c] = s * (1.0f / RF_BLOCK);
}

__global__ void __launch_bounds__(kPermThreads) unpermute_kernel(const uint16_t* __restrict__ o_int, int layout, int B,
                                                                 int S, int N, rf_plan_t g,
                                                                 uint16_t* __restrict__ out) {
  const int tile = blockIdx.x;
  const int bn = blockIdx.y;
  const int b = bn / N, n = bn - b * N;
  const int chunk = threadIdx.x & 15;
  const int rsub = threadIdx.x >> 4;
  const int64_t src_base = ((int64_t)bn * g.S_int + (int64_t)tile * RF_BLOCK) * RF_HEAD_DIM + chunk * 8;
  uint4 buf[kPasses];
#pragma unroll
  for (int p = 0; p < kPasses; ++p)
    buf[p] = __ldcs(reinterpret_cast<const uint4*>(o_int + src_base + (int64_t)(p * kRowsPerPass + rsub) * RF_HEAD_DIM));
#pragma unroll
  for (int p = 0; p < kPasses; ++p) {
    const int s = rf_src_of_row(g, tile * RF_BLOCK + p * kRowsPerPass + rsub);
    if (s >= 0) *reinterpret_cast<uint4*>(out + rf_token_offset(layout, B, S, N, b, n, s) + chunk * 8) = buf[p];
  }
}

}  // namespace

cudaError_t launch_permute_pool(const void* q, const void* k, const void* v, int dtype, int layout, int B, int S,
                                int Sk, int N, const rf_plan_t& g, const rf_plan_t& gk, void* q_int, void* k_int,
                                void* v_int, float* pooled_q, float* pooled_k, cudaStream_t stream) {
  auto kern = dtype == RF_F16 ? permute_pool_kernel<true> : permute_pool_kernel<false>;
  auto s16 = [](const void* x) { return static_cast<const uint16_t*>(x); };
  auto d16 = [](void* x) { return static_cast<uint16_t*>(x); };
  PermArgs a{};
  if (S == Sk && std::memcmp(&g, &gk, sizeof(rf_plan_t)) == 0) {   // one geometry: one pass over q, k, v
    a = PermArgs{{s16(q), s16(k), s16(v)}, {d16(q_int), d16(k_int), d16(v_int)}, {pooled_q, pooled_k}, 3};
    kern<<<dim3(g.n_tiles, B * N), kPermThreads, 0, stream>>>(a, layout, B, S, N, g);
    return cudaGetLastError();
  }
  a = PermArgs{{s16(q), nullptr, nullptr}, {d16(q_int), nullptr, nullptr}, {pooled_q, nullptr}, 1};
  kern<<<dim3(g.n_tiles, B * N), kPermThreads, 0, stream>>>(a, layout, B, S, N, g);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  a = PermArgs{{s16(k), s16(v), nullptr}, {d16(k_int), d16(v_int), nullptr}, {pooled_k, nullptr}, 2};
  kern<<<dim3(gk.n_tiles, B * N), kPermThreads, 0, stream>>>(a, layout, B, Sk, N, gk);
  return cudaGetLastError();
}

cudaError_t launch_unpermute(const void* o_int, int layout, int B, int S, int N, const rf_plan_t& g, void* out,
                             cudaStream_t stream) {
  dim3 grid(g.n_tiles, B * N);
  unpermute_kernel<<<grid, kPermThreads, 0, stream>>>(static_cast<const uint16_t*>(o_int), layout, B, S, N, g,
                                                      static_cast<uint16_t*>(out));
  return cudaGetLastError();
}

}  // namespace rf
