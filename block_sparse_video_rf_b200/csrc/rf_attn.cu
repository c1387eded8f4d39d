// Block-sparse flash attention on sm_100a tensor cores (K3).
//
// lite_boost.ops.sparse_attention, rf_v2 pipeline: rain_fusion_attention
// over the kept KV blocks, then the inverse reorder (fused here: each output
// row is written straight to its token's place in the caller's layout).
// vllm-omni "RainFusion Attention", intro: prefix rows and first-frame
// blocks stay dense; every other query block attends to its highest-scoring
// key blocks.
//
// Work unit: one 128-row query tile of one (b, head).  Its KV list is every
// prefix tile, then either every sparse block (dense tile) or the blocks set
// in its mask row, in ascending order.  Persistent CTAs (two per SM) take
// units from a global counter in (head, tile) order, dense tiles of a head
// first, so the heads in flight keep their K/V in L2.
//
// CTA = 6 warps:
//   warps 0-3  softmax: thread t owns query row t (TMEM lane t); online
//              softmax in exp2 with a lazily updated running max, P written
//              back to TMEM as bf16, epilogue O / l -> bf16 -> global.
//   warp 4     TMA producer (one thread): Q tile, then K and V tiles of the
//              KV list, 128-byte swizzled boxes of 128 rows x 64 columns.
//   warp 5     MMA issuer (one thread) and TMEM owner:
//              S = Q K^T   (tcgen05 kind::f16, A/B from shared memory)
//              O += P V    (A = P from tensor memory, B = V MN-major)
// Tensor memory (256 columns): S fp32 in [0, 128), aliased by P bf16 in
// [0, 64); O fp32 in [128, 256).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math_constants.h>

#include <algorithm>

#include "rf_geometry.h"
#include "rf_kernels.h"
#include "sm100_ptx.cuh"

namespace rf {

namespace {

constexpr int kThreads = 192;
constexpr int kSoftmaxThreads = 128;
constexpr int kTileBytes = RF_BLOCK * RF_HEAD_DIM * 2;   // 32 KB
constexpr int kHalfBytes = kTileBytes / 2;               // 64 columns x 128 rows
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kColS = 0, kColO = 128;
constexpr float kRescaleThreshold = 8.0f;                // log2 units
constexpr uint64_t kWaitLimitNs = 2000000000ull;

struct Item {
  int bn, qt, ntiles, pad;
};

struct __align__(1024) Smem {
  uint8_t q[kTileBytes];
  uint8_t k[kTileBytes];
  uint8_t v[kTileBytes];
  uint64_t q_full, q_empty, k_full, k_empty, v_full, v_empty;
  uint64_t s_full, p_full, pv_done, o_empty;
  uint64_t item_full[2], item_empty[2];
  Item items[2];
  uint32_t tmem_base;
  int abort;
};

struct AttnParams {
  rf_plan_t g;
  int B, S, N, layout;
  int total_items;
  int n_ptiles;      // prefix tiles (P_pad / 128)
  int p_rem;         // valid rows of the last prefix tile when it is partial, else 0
  float scale_log2;
  const uint32_t* mask;
  int* counter;
  int* status;
  __nv_bfloat16* out;
};

__device__ __forceinline__ bool is_dense_tile(const AttnParams& p, int qt) {
  return p.g.dense || qt < p.n_ptiles || (qt - p.n_ptiles) < p.g.ff;
}

// ---------------------------------------------------------------- producer
__device__ void producer_loop(Smem& sm, const AttnParams& p, const CUtensorMap* tq, const CUtensorMap* tk,
                              const CUtensorMap* tv) {
  volatile int* abort = &sm.abort;
  const uint64_t pol_q = l2_policy_evict_first();
  const uint64_t pol_kv = l2_policy_evict_last();
  uint32_t it = 0, nq = 0, nk = 0, nv = 0;
  const int S_int = p.g.S_int;
  bool ok = true;

  auto load_kv = [&](int row) -> bool {
    if (nk > 0 && !rf_wait(&sm.k_empty, (nk - 1) & 1, abort, p.status, RF_ERR_TIMEOUT, kWaitLimitNs)) return false;
    mbar_arrive_expect_tx(&sm.k_full, kTileBytes);
    tma_load_2d(sm.k, tk, &sm.k_full, 0, row, pol_kv);
    tma_load_2d(sm.k + kHalfBytes, tk, &sm.k_full, 64, row, pol_kv);
    ++nk;
    if (nv > 0 && !rf_wait(&sm.v_empty, (nv - 1) & 1, abort, p.status, RF_ERR_TIMEOUT, kWaitLimitNs)) return false;
    mbar_arrive_expect_tx(&sm.v_full, kTileBytes);
    tma_load_2d(sm.v, tv, &sm.v_full, 0, row, pol_kv);
    tma_load_2d(sm.v + kHalfBytes, tv, &sm.v_full, 64, row, pol_kv);
    ++nv;
    return true;
  };

  while (ok) {
    const int w = atomicAdd(p.counter, 1);
    const int slot = it & 1;
    if (it >= 2 && !rf_wait(&sm.item_empty[slot], ((it >> 1) - 1) & 1, abort, p.status, RF_ERR_TIMEOUT,
                            kWaitLimitNs)) {
      ok = false;
      break;
    }
    Item itm{-1, 0, 0, 0};
    const uint32_t* mrow = nullptr;
    bool dense = true;
    if (w < p.total_items) {
      itm.bn = w / p.g.n_tiles;
      itm.qt = w - itm.bn * p.g.n_tiles;
      dense = is_dense_tile(p, itm.qt);
      if (dense) {
        itm.ntiles = p.g.n_tiles;
      } else {
        mrow = p.mask + ((size_t)itm.bn * p.g.nb + (itm.qt - p.n_ptiles)) * p.g.mask_words;
        int cnt = 0;
        for (int wd = 0; wd < p.g.mask_words; ++wd) cnt += __popc(mrow[wd]);
        itm.ntiles = p.n_ptiles + cnt;
      }
    }
    sm.items[slot] = itm;
    mbar_arrive(&sm.item_full[slot]);
    ++it;
    if (itm.bn < 0) break;

    const int base = itm.bn * S_int;
    if (nq > 0 && !rf_wait(&sm.q_empty, (nq - 1) & 1, abort, p.status, RF_ERR_TIMEOUT, kWaitLimitNs)) {
      ok = false;
      break;
    }
    mbar_arrive_expect_tx(&sm.q_full, kTileBytes);
    tma_load_2d(sm.q, tq, &sm.q_full, 0, base + itm.qt * RF_BLOCK, pol_q);
    tma_load_2d(sm.q + kHalfBytes, tq, &sm.q_full, 64, base + itm.qt * RF_BLOCK, pol_q);
    ++nq;

    for (int t = 0; t < p.n_ptiles && ok; ++t) ok = load_kv(base + t * RF_BLOCK);
    if (dense) {
      for (int j = 0; j < p.g.nb && ok; ++j) ok = load_kv(base + (p.n_ptiles + j) * RF_BLOCK);
    } else {
      for (int wd = 0; wd < p.g.mask_words && ok; ++wd) {
        uint32_t bits = mrow[wd];
        while (bits && ok) {
          const int j = 32 * wd + __ffs(bits) - 1;
          bits &= bits - 1;
          ok = load_kv(base + (p.n_ptiles + j) * RF_BLOCK);
        }
      }
    }
  }
  if (!ok) {
    // Let the copies already issued land before the CTA may exit.
    if (nq > 0) rf_wait(&sm.q_full, (nq - 1) & 1, abort, p.status, RF_ERR_TIMEOUT, kWaitLimitNs / 4);
    if (nk > 0) rf_wait(&sm.k_full, (nk - 1) & 1, abort, p.status, RF_ERR_TIMEOUT, kWaitLimitNs / 4);
    if (nv > 0) rf_wait(&sm.v_full, (nv - 1) & 1, abort, p.status, RF_ERR_TIMEOUT, kWaitLimitNs / 4);
  }
}

// ---------------------------------------------------------------- MMA issuer
__device__ void mma_loop(Smem& sm, const AttnParams& p, uint32_t tmem) {
  volatile int* abort = &sm.abort;
  constexpr uint32_t idesc_qk = make_idesc_bf16(128, 128, false);
  constexpr uint32_t idesc_pv = make_idesc_bf16(128, 128, true);
  const uint32_t q_addr = smem_u32(sm.q), k_addr = smem_u32(sm.k), v_addr = smem_u32(sm.v);
  uint32_t it = 0, nq = 0, nk = 0, nv = 0, np = 0, npv = 0, items_done = 0;
  for (;;) {
    const int slot = it & 1;
    if (!rf_wait(&sm.item_full[slot], (it >> 1) & 1, abort, p.status, RF_ERR_TIMEOUT, kWaitLimitNs)) return;
    const Item itm = sm.items[slot];
    mbar_arrive(&sm.item_empty[slot]);
    ++it;
    if (itm.bn < 0) return;
    if (!rf_wait(&sm.q_full, nq & 1, abort, p.status, RF_ERR_TIMEOUT, kWaitLimitNs)) return;
    ++nq;
    for (int j = 0; j < itm.ntiles; ++j) {
      if (!rf_wait(&sm.k_full, nk & 1, abort, p.status, RF_ERR_TIMEOUT, kWaitLimitNs)) return;
      ++nk;
      // P of the previous tile lives in the S columns: its P*V must be done.
      if (npv > 0 && !rf_wait(&sm.pv_done, (npv - 1) & 1, abort, p.status, RF_ERR_TIMEOUT, kWaitLimitNs)) return;
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint32_t off = (kk >> 2) * kHalfBytes + (kk & 3) * 32;
        mma_ss(tmem + kColS, make_sdesc_sw128(q_addr + off, 16, 1024), make_sdesc_sw128(k_addr + off, 16, 1024),
               idesc_qk, kk > 0);
      }
      mma_commit(&sm.s_full);
      mma_commit(&sm.k_empty);
      if (j == itm.ntiles - 1) mma_commit(&sm.q_empty);

      if (!rf_wait(&sm.p_full, np & 1, abort, p.status, RF_ERR_TIMEOUT, kWaitLimitNs)) return;
      ++np;
      if (!rf_wait(&sm.v_full, nv & 1, abort, p.status, RF_ERR_TIMEOUT, kWaitLimitNs)) return;
      ++nv;
      if (j == 0 && items_done > 0 &&
          !rf_wait(&sm.o_empty, (items_done - 1) & 1, abort, p.status, RF_ERR_TIMEOUT, kWaitLimitNs))
        return;
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        mma_ts(tmem + kColO, tmem + kColS + kk * 8, make_sdesc_sw128(v_addr + kk * 2048, kHalfBytes, 1024), idesc_pv,
               (j > 0 || kk > 0) ? 1u : 0u);
      }
      mma_commit(&sm.pv_done);
      mma_commit(&sm.v_empty);
      ++npv;
    }
    ++items_done;
  }
}

// ---------------------------------------------------------------- softmax + epilogue
__device__ void softmax_loop(Smem& sm, const AttnParams& p, uint32_t tmem) {
  volatile int* abort = &sm.abort;
  const int row = threadIdx.x;                 // 0..127 == TMEM lane
  const int warp = row >> 5;
  const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16);
  const uint32_t tS = lane_base + kColS, tO = lane_base + kColO;
  const float sl2 = p.scale_log2;
  uint32_t it = 0, ns = 0, npv = 0;
  for (;;) {
    const int slot = it & 1;
    if (!rf_wait(&sm.item_full[slot], (it >> 1) & 1, abort, p.status, RF_ERR_TIMEOUT, kWaitLimitNs)) return;
    const Item itm = sm.items[slot];
    mbar_arrive(&sm.item_empty[slot]);
    ++it;
    if (itm.bn < 0) return;

    float m_use = -CUDART_INF_F, l = 0.f;
    for (int j = 0; j < itm.ntiles; ++j) {
      if (!rf_wait(&sm.s_full, ns & 1, abort, p.status, RF_ERR_TIMEOUT, kWaitLimitNs)) return;
      ++ns;
      tc_fence_after();
      uint32_t s[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(tS + 32 * c, s[c]);
      tmem_wait_ld();
#pragma unroll
      for (int c = 0; c < 4; ++c) reg_fence32(s[c]);

      if (p.p_rem != 0 && j == p.n_ptiles - 1) {
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int e = 0; e < 32; ++e)
            if (32 * c + e >= p.p_rem) s[c][e] = __float_as_uint(-CUDART_INF_F);
      }
      float mx = -CUDART_INF_F;
#pragma unroll
      for (int c = 0; c < 4; ++c)
#pragma unroll
        for (int e = 0; e < 32; ++e) mx = fmaxf(mx, __uint_as_float(s[c][e]));
      const float mx_s = mx * sl2;
      float alpha = 1.f;
      bool rescale = false;
      if (j == 0) {
        m_use = mx_s;
      } else if (mx_s > m_use + kRescaleThreshold) {
        alpha = ex2_approx(m_use - mx_s);
        m_use = mx_s;
        rescale = true;
      }
      // exponentials, packed to bf16 pairs in place (s[c][0..15] of each chunk)
      float sum = 0.f;
      uint32_t pk[64];
#pragma unroll
      for (int c = 0; c < 4; ++c)
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          const float p0 = ex2_approx(fmaf(__uint_as_float(s[c][e]), sl2, -m_use));
          const float p1 = ex2_approx(fmaf(__uint_as_float(s[c][e + 1]), sl2, -m_use));
          sum += p0 + p1;
          pk[16 * c + e / 2] = pack_bf16x2(p0, p1);
        }
      l = l * alpha + sum;
      if (__any_sync(0xFFFFFFFFu, rescale)) {
        // O holds the sum over the tiles before j (their P*V completed before
        // this tile's S was computed).
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t o[32];
          tmem_ld32(tO + 32 * c, o);
          tmem_wait_ld();
          reg_fence32(o);
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
          tmem_st32(tO + 32 * c, o);
        }
      }
      tmem_st32(tS, *reinterpret_cast<uint32_t(*)[32]>(&pk[0]));
      tmem_st32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&pk[32]));
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&sm.p_full);
      ++npv;
    }

    // epilogue: wait for the last P*V of this tile
    if (!rf_wait(&sm.pv_done, (npv - 1) & 1, abort, p.status, RF_ERR_TIMEOUT, kWaitLimitNs)) return;
    tc_fence_after();
    const float rl = 1.f / l;
    const int b = itm.bn / p.N, n = itm.bn - b * p.N;
    const int src = rf_src_of_row(p.g, itm.qt * RF_BLOCK + row);
    __nv_bfloat16* dst = src >= 0 ? p.out + rf_token_offset(p.layout, p.B, p.S, p.N, b, n, src) : nullptr;
#pragma unroll 1
    for (int c = 0; c < 4; ++c) {
      uint32_t o[32];
      tmem_ld32(tO + 32 * c, o);
      tmem_wait_ld();
      reg_fence32(o);
      uint32_t w[16];
#pragma unroll
      for (int e = 0; e < 16; ++e)
        w[e] = pack_bf16x2(__uint_as_float(o[2 * e]) * rl, __uint_as_float(o[2 * e + 1]) * rl);
      if (dst) {
        uint4* d4 = reinterpret_cast<uint4*>(dst + 32 * c);
#pragma unroll
        for (int e = 0; e < 4; ++e) d4[e] = make_uint4(w[4 * e], w[4 * e + 1], w[4 * e + 2], w[4 * e + 3]);
      }
    }
    tc_fence_before();
    mbar_arrive(&sm.o_empty);
  }
}

__global__ void __launch_bounds__(kThreads, 2)
    attn_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const AttnParams p) {
  extern __shared__ uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(&sm.q_full, 1);
    mbar_init(&sm.q_empty, 1);
    mbar_init(&sm.k_full, 1);
    mbar_init(&sm.k_empty, 1);
    mbar_init(&sm.v_full, 1);
    mbar_init(&sm.v_empty, 1);
    mbar_init(&sm.s_full, 1);
    mbar_init(&sm.p_full, kSoftmaxThreads);
    mbar_init(&sm.pv_done, 1);
    mbar_init(&sm.o_empty, kSoftmaxThreads);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sm.item_full[i], 1);
      mbar_init(&sm.item_empty[i], kSoftmaxThreads + 1);
    }
    sm.abort = 0;
    fence_mbar_init();
  }
  if (warp == 4 && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  if (warp == 5) {
    tmem_alloc(&sm.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;

  if (warp < 4) {
    softmax_loop(sm, p, tmem);
  } else if (warp == 4) {
    if (lane == 0) producer_loop(sm, p, &tm_q, &tm_k, &tm_v);
  } else {
    if (lane == 0) mma_loop(sm, p, tmem);
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 5) tmem_dealloc(tmem, kTmemCols);
}

// ---------------------------------------------------------------- host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult qres;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &qres) == cudaSuccess &&
        qres == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

// [rows, 128] bf16 row-major, boxes of 128 rows x 64 columns, 128-byte swizzle.
bool make_tile_map(CUtensorMap* map, const void* base, uint64_t rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[2] = {RF_HEAD_DIM, rows};
  const cuuint64_t strides[1] = {RF_HEAD_DIM * 2};
  const cuuint32_t box[2] = {64, RF_BLOCK};
  const cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

cudaError_t launch_attention(const void* q_int, const void* k_int, const void* v_int, const uint32_t* mask,
                             int layout, int B, int S, int N, const rf_plan_t& g, float scale, void* out,
                             int* counter, int* status, cudaStream_t stream) {
  const uint64_t rows = (uint64_t)B * N * g.S_int;
  CUtensorMap tq, tk, tv;
  if (!make_tile_map(&tq, q_int, rows) || !make_tile_map(&tk, k_int, rows) || !make_tile_map(&tv, v_int, rows))
    return cudaErrorInvalidValue;
  AttnParams p;
  p.g = g;
  p.B = B;
  p.S = S;
  p.N = N;
  p.layout = layout;
  p.total_items = B * N * g.n_tiles;
  p.n_ptiles = g.P_pad / RF_BLOCK;
  p.p_rem = g.P % RF_BLOCK;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.mask = mask;
  p.counter = counter;
  p.status = status;
  p.out = static_cast<__nv_bfloat16*>(out);

  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  const size_t smem = sizeof(Smem) + 1024;
  e = cudaFuncSetAttribute(attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  e = cudaMemsetAsync(counter, 0, sizeof(int), stream);
  if (e != cudaSuccess) return e;
  const int grid = std::min(2 * sms, p.total_items);
  attn_kernel<<<grid, kThreads, smem, stream>>>(tq, tk, tv, p);
  return cudaGetLastError();
}

}  // namespace rf
