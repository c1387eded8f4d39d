// Token reorder with block pooling fused in (K1), and the inverse reorder
// (K4): row gathers/scatters of 256-byte rows, bound by HBM (K1's fp8 form,
// which also converts every value, by its instruction issue).
//
// lite_boost.ops.sparse_attention, rf_v2 pipeline: token reorder, then block
// pooling; inverse reorder at the end.  vllm-omni "RainFusion Attention":
// 128-token key blocks are pooled (intro); the reorder groups video tokens
// into 8x8 tiles and promotes the non-aligned rest ("Geometry handling").
//
// At the fp8 precision (lite_boost.ops.sparse_attention lists one; the pages
// fix no scaling rule) K1 writes the reordered tiles as e4m3 codes instead
// of 16-bit copies.  The reading taken: one fp32 scale per 128-row tile of
// the internal layout, per tensor and head (the attention's own tile),
// scale = amax(|x|) / 448 with 448 the largest finite e4m3 value, code =
// e4m3 round-to-nearest-even, saturating, of x * (448 / amax) in fp32; an
// all-zero tile has scale 0 and codes 0.  V's tiles are stored transposed
// (channel-major) so that the P V product reads them K-major, and vmax[head]
// is the largest V tile scale of the head.
#include <cuda_runtime.h>

#include <cstring>

#include "rf_dtype.h"
#include "rf_geometry.h"
#include "rf_kernels.h"
#include "sm100_ptx.cuh"

namespace rf {

namespace {

constexpr int kPermThreads = 256;   // 16 rows x 16 chunks of 16 bytes per pass
constexpr int kRowsPerPass = kPermThreads / 16;
constexpr int kPasses = RF_BLOCK / kRowsPerPass;

// Token (sequence index) of each of a thread's rows of internal tile `tile`
// (row p * kRowsPerPass + rsub; -1 for a pad row): a sparse block's rows
// from its two 8x8 tiles (two divisions for the block), prefix rows one by
// one.
__device__ __forceinline__ void tile_sources(const rf_plan_t& g, int tile, int rsub, int (&src)[kPasses]) {
  if (!g.dense && tile * RF_BLOCK >= g.P_pad) {
    const RfBlockTiles bt = rf_block_tiles(g, tile - g.P_pad / RF_BLOCK);
#pragma unroll
    for (int p = 0; p < kPasses; ++p) src[p] = rf_src_in_block(g, bt, p * kRowsPerPass + rsub);
  } else {
#pragma unroll
    for (int p = 0; p < kPasses; ++p) src[p] = rf_src_of_row(g, tile * RF_BLOCK + p * kRowsPerPass + rsub);
  }
}

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

  int tok[kPasses];
  tile_sources(g, tile, rsub, tok);
  int64_t src_off[kPasses];
#pragma unroll
  for (int p = 0; p < kPasses; ++p)
    src_off[p] = tok[p] < 0 ? -1 : rf_token_offset(layout, B, S, N, b, n, tok[p]) + chunk * 8;
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
  float* pooled = t == 0 ? a.pooled[0] : a.pooled[1];   // constant indices: no local copy of the arguments
  if (!pooled) return;
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < kRowsPerPass; ++i) s += red[t][i][c];
  const int blk = tile - g.P_pad / RF_BLOCK;
  pooled[((int64_t)bn * g.nb + blk) * RF_HEAD_DIM + c] = s * (1.0f / RF_BLOCK);
}

// fp8 form: e4m3 codes and tile scales in place of the 16-bit copies.

struct PermArgs8 {
  const uint16_t* src[3];
  uint8_t* dst[3];    // e4m3 codes, internal layout (the v_index tensor's tiles transposed)
  float* scales[3];   // [BN, n_tiles] tile scales of each tensor
  float* pooled[2];   // block means of tensors 0 and 1 (nullptr: not pooled)
  int count;          // tensors in use
  int v_index;        // the transposed tensor, whose largest tile scale goes to vmax (-1: none)
  float* vmax;        // [BN], zero before the launch
};

// One CTA = one 128-row internal tile of one (b, head), for each tensor in
// turn: its rows gathered (8 16-byte loads in flight per thread), the tile's
// amax behind one barrier, then its codes.  Few registers, so that several
// CTAs share an SM and hide the barriers.  Block means as permute_pool_kernel,
// summed in the same order.
template <bool kF16>
__global__ void __launch_bounds__(kPermThreads, 3) permute_pool_fp8_kernel(PermArgs8 a, int layout, int B, int S,
                                                                           int N, rf_plan_t g) {
  __shared__ float red[2][kRowsPerPass][RF_HEAD_DIM];
  __shared__ float red_max[3][kPermThreads / 32];
  __shared__ __align__(16) uint32_t vr[RF_BLOCK][RF_HEAD_DIM / 4];   // V's codes, row-major, words swizzled
  const int tile = blockIdx.x;
  const int bn = blockIdx.y;
  const int b = bn / N, n = bn - b * N;
  const int chunk = threadIdx.x & 15;     // 16-byte column chunk
  const int rsub = threadIdx.x >> 4;      // row within the pass
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool sparse = (tile * RF_BLOCK >= g.P_pad) && !g.dense;
  int src[kPasses];   // token of each of the thread's rows (-1: pad row)
  tile_sources(g, tile, rsub, src);
  const int64_t code_base = ((int64_t)bn * g.S_int + (int64_t)tile * RF_BLOCK) * RF_HEAD_DIM;
  // every tensor's rows requested into L2 at once (one request per 128-byte
  // line, no registers held), so that the tile's DRAM reads overlap the
  // tensor-by-tensor work below
  if ((chunk & 7) == 0) {
#pragma unroll
    for (int t = 0; t < 3; ++t) {
      if (t >= a.count) break;
      const uint16_t* in = t == 0 ? a.src[0] : t == 1 ? a.src[1] : a.src[2];
#pragma unroll
      for (int p = 0; p < kPasses; ++p)
        if (src[p] >= 0) prefetch_l2(in + rf_token_offset(layout, B, S, N, b, n, src[p]) + chunk * 8);
    }
  }

#pragma unroll 1
  for (int t = 0; t < a.count; ++t) {
    // the tensor's pointers, chosen with constant indices (a runtime index
    // into the parameter arrays would copy them to local memory)
    const uint16_t* in = t == 0 ? a.src[0] : t == 1 ? a.src[1] : a.src[2];
    uint8_t* codes = t == 0 ? a.dst[0] : t == 1 ? a.dst[1] : a.dst[2];
    float* scales = t == 0 ? a.scales[0] : t == 1 ? a.scales[1] : a.scales[2];
    float* pooled = t == 0 ? a.pooled[0] : t == 1 ? a.pooled[1] : nullptr;
    uint4 buf[kPasses];
#pragma unroll
    for (int p = 0; p < kPasses; ++p)
      buf[p] = src[p] < 0 ? make_uint4(0, 0, 0, 0)
                          : __ldcs(reinterpret_cast<const uint4*>(
                                in + rf_token_offset(layout, B, S, N, b, n, src[p]) + chunk * 8));
    // amax on the packed values: for finite bf16 and fp16 alike, |x| orders
    // like the integer bits & 0x7FFF, so a per-half unsigned max finds it
    // exactly (nothing unpacked stays live across the barrier)
    uint32_t m2 = 0;
#pragma unroll
    for (int p = 0; p < kPasses; ++p) {
      m2 = __vmaxu2(m2, __vmaxu2(buf[p].x & 0x7FFF7FFFu, buf[p].y & 0x7FFF7FFFu));
      m2 = __vmaxu2(m2, __vmaxu2(buf[p].z & 0x7FFF7FFFu, buf[p].w & 0x7FFF7FFFu));
    }
    const uint32_t mbits = max(m2 & 0xFFFFu, m2 >> 16);
    float amax;
    if (kF16)
      amax = __half2float(__ushort_as_half((unsigned short)mbits));
    else
      amax = __uint_as_float(mbits << 16);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
    if (lane == 0) red_max[t][warp] = amax;
    __syncthreads();
    amax = red_max[t][0];
#pragma unroll
    for (int i = 1; i < kPermThreads / 32; ++i) amax = fmaxf(amax, red_max[t][i]);
    const float inv = amax > 0.f ? __fdiv_rn(448.f, amax) : 0.f;
    const float scale = __fdiv_rn(amax, 448.f);
    const bool transposed = t == a.v_index;
    const bool pool = sparse && pooled;
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};   // the block means' partial sums
    const uint64_t inv2 = f2_pack(inv, inv);
#pragma unroll
    for (int p = 0; p < kPasses; ++p) {
      if (pool) acc_half8<kF16>(acc, buf[p]);
      float f[8];
      unpack_half8<kF16>(buf[p], f);
      const int r = p * kRowsPerPass + rsub;
      float y[8];
#pragma unroll
      for (int i = 0; i < 8; i += 2) f2_unpack(f2_mul(f2_pack(f[i], f[i + 1]), inv2), y[i], y[i + 1]);
      const uint32_t lo = pack_e4m3x4(y[0], y[1], y[2], y[3]);
      const uint32_t hi = pack_e4m3x4(y[4], y[5], y[6], y[7]);
      if (!transposed) {
        *reinterpret_cast<uint2*>(codes + code_base + (int64_t)r * RF_HEAD_DIM + chunk * 8) = make_uint2(lo, hi);
      } else {
        // row r's 8 codes at logical words 2 chunk, 2 chunk + 1, the pair
        // moved by an even swizzle of its row group (conflict-free here,
        // 2-way in the transposing read below)
        *reinterpret_cast<uint2*>(&vr[r][(2 * chunk) ^ (2 * ((r >> 2) & 15))]) = make_uint2(lo, hi);
      }
    }
    if (pool) {
#pragma unroll
      for (int i = 0; i < 8; ++i) red[t][rsub][chunk * 8 + i] = acc[i];
    }
    if (threadIdx.x == 0) {
      scales[(int64_t)bn * g.n_tiles + tile] = scale;
      // non-negative floats order like their bit patterns
      if (transposed) atomicMax(reinterpret_cast<int*>(a.vmax) + bn, __float_as_int(scale));
    }
  }
  __syncthreads();   // the transposed V tile and the block means' partial sums are in place
  if (a.v_index >= 0) {
    // the transposed V tile, 128 channel rows of 128 bytes: a thread takes
    // rows 4 l .. 4 l + 3 (l its lane) of channel quads warp + 8 k, and
    // transposes each 4 x 4 block of bytes in registers; a warp then writes
    // 128 contiguous bytes of one channel per store
    uint8_t* codes = a.v_index == 1 ? a.dst[1] : a.dst[2];
    const int sw = 2 * (lane & 15);
#pragma unroll
    for (int kk = 0; kk < RF_HEAD_DIM / 4 / (kPermThreads / 32); ++kk) {
      const int cq = warp + (kPermThreads / 32) * kk;
      uint32_t w[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) w[j] = vr[4 * lane + j][cq ^ sw];
      const uint32_t t0 = __byte_perm(w[0], w[1], 0x5140), t1 = __byte_perm(w[0], w[1], 0x7362);
      const uint32_t t2 = __byte_perm(w[2], w[3], 0x5140), t3 = __byte_perm(w[2], w[3], 0x7362);
      const uint32_t o[4] = {__byte_perm(t0, t2, 0x5410), __byte_perm(t0, t2, 0x7632), __byte_perm(t1, t3, 0x5410),
                             __byte_perm(t1, t3, 0x7632)};
#pragma unroll
      for (int i = 0; i < 4; ++i)
        *reinterpret_cast<uint32_t*>(codes + code_base + (int64_t)(4 * cq + i) * RF_BLOCK + 4 * lane) = o[i];
    }
  }
  if (!sparse) return;
  const int t = threadIdx.x >> 7, c = threadIdx.x & 127;
  float* pooled = t == 0 ? a.pooled[0] : a.pooled[1];
  if (t >= a.count || !pooled) return;
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < kRowsPerPass; ++i) s += red[t][i][c];
  const int blk = tile - g.P_pad / RF_BLOCK;
  pooled[((int64_t)bn * g.nb + blk) * RF_HEAD_DIM + c] = s * (1.0f / RF_BLOCK);
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
  int src[kPasses];
  tile_sources(g, tile, rsub, src);
#pragma unroll
  for (int p = 0; p < kPasses; ++p)
    if (src[p] >= 0) *reinterpret_cast<uint4*>(out + rf_token_offset(layout, B, S, N, b, n, src[p]) + chunk * 8) = buf[p];
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

cudaError_t launch_permute_pool_fp8(const void* q, const void* k, const void* v, int dtype, int layout, int B, int S,
                                    int Sk, int N, const rf_plan_t& g, const rf_plan_t& gk, uint8_t* q8, uint8_t* k8,
                                    uint8_t* v8, float* scales, float* vmax, float* pooled_q, float* pooled_k,
                                    cudaStream_t stream) {
  const int BN = B * N;
  cudaError_t e = cudaMemsetAsync(vmax, 0, sizeof(float) * BN, stream);
  if (e != cudaSuccess) return e;
  auto kern = dtype == RF_F16 ? permute_pool_fp8_kernel<true> : permute_pool_fp8_kernel<false>;
  auto s16 = [](const void* x) { return static_cast<const uint16_t*>(x); };
  float* sq = scales;
  float* sk = sq + (size_t)BN * g.n_tiles;
  float* sv = sk + (size_t)BN * gk.n_tiles;
  if (S == Sk && std::memcmp(&g, &gk, sizeof(rf_plan_t)) == 0) {   // one geometry: one pass over q, k, v
    const PermArgs8 a{{s16(q), s16(k), s16(v)}, {q8, k8, v8}, {sq, sk, sv}, {pooled_q, pooled_k}, 3, 2, vmax};
    kern<<<dim3(g.n_tiles, BN), kPermThreads, 0, stream>>>(a, layout, B, S, N, g);
    return cudaGetLastError();
  }
  const PermArgs8 aq{{s16(q), nullptr, nullptr}, {q8, nullptr, nullptr}, {sq, nullptr, nullptr},
                     {pooled_q, nullptr}, 1, -1, vmax};
  kern<<<dim3(g.n_tiles, BN), kPermThreads, 0, stream>>>(aq, layout, B, S, N, g);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const PermArgs8 akv{{s16(k), s16(v), nullptr}, {k8, v8, nullptr}, {sk, sv, nullptr}, {pooled_k, nullptr}, 2, 1,
                      vmax};
  kern<<<dim3(gk.n_tiles, BN), kPermThreads, 0, stream>>>(akv, layout, B, Sk, N, gk);
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
