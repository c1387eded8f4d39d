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
// in its mask row, in ascending order.  Persistent CTAs (one per SM) take
// units from a global counter in (head, tile) order, dense tiles of a head
// first, so the heads in flight keep their K/V in L2.
//
// CTA = 10 warps, software-pipelined over the KV list:
//   warps 0-7  softmax: warps w and w + 4 share query rows 32 (w % 4) ..
//              32 (w % 4) + 31 (TMEM lanes) and split the 128 key columns in
//              halves; the row max and the row sum are combined through
//              shared memory.  Online softmax in exp2 with a lazily updated
//              running max.  Most exponentials run on the MUFU unit, one
//              pair in four on the FMA pipe (polynomial).  At the end of a
//              unit the same threads write O / l -> bf16 -> the caller's
//              layout while the tensor pipe starts the next unit.
//   warp 8     TMA producer (one thread): Q tile, K and V tiles of the KV
//              list through 3- and 2-stage rings of 128-byte swizzled boxes
//              (128 rows x 64 columns), K two tiles ahead of V.
//   warp 9     MMA issuer (one thread) and TMEM owner:
//              S = Q K^T   (tcgen05 kind::f16, A/B from shared memory)
//              O += P V    (A = P from tensor memory, B = V MN-major)
// Tensor memory (512 columns): S0 [0,128), S1 [128,256) double-buffer the
// score tile; O [256,384) is the accumulator; P0 [384,448), P1 [448,512)
// double-buffer P as bf16.  The QK of tile j+2 only waits for the softmax to
// have read S of tile j, so the tensor pipe runs S = Q K^T of later tiles
// while the softmax of tile j is still computing.
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

constexpr int kThreads = 320;
constexpr int kSoftmaxThreads = 256;
constexpr int kKStages = 3;                              // K ring depth
constexpr int kVStages = 2;                              // V ring depth
constexpr int kKAhead = 2;                               // K tiles issued ahead of V
constexpr int kTileBytes = RF_BLOCK * RF_HEAD_DIM * 2;   // 32 KB
constexpr int kHalfBytes = kTileBytes / 2;               // 64 columns x 128 rows
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0, kColO = 256, kColP = 384;  // S b at 128 b; P b at 384 + 64 b
constexpr int kPolyEvery = 4;                            // pair i uses the polynomial when i % 4 == 3
constexpr float kRescaleThreshold = 8.0f;                // log2 units
constexpr uint64_t kWaitLimitNs = 2000000000ull;

struct Item {
  int bn, qt, ntiles, pad;
};

struct __align__(1024) Smem {
  uint8_t q[kTileBytes];
  uint8_t k[kKStages][kTileBytes];
  uint8_t v[kVStages][kTileBytes];
  uint64_t q_full, q_empty;
  uint64_t k_full[kKStages], k_empty[kKStages], v_full[kVStages], v_empty[kVStages];
  uint64_t s_full[2], s_read[2], p_full[2], p_free[2];
  uint64_t o_full, o_empty;
  uint64_t drain;               // MMA issuer's last commit when it leaves early
  uint64_t xbar[4];             // per row quadrant: rendezvous of its two softmax warps
  uint64_t item_full[2], item_empty[2];
  Item items[2];
  float xmax[2][2][RF_BLOCK];   // [tile parity][column half][row] partial row maxima
  float xsum[2][RF_BLOCK];      // [column half][row] partial row sums at the end of a unit
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
  uint64_t wait_limit_ns;   // limit of every device-side wait
  int skip_first_q;         // test control: the first unit's Q load is never issued
};

__device__ __forceinline__ bool is_dense_tile(const AttnParams& p, int qt) {
  return p.g.dense || qt < p.n_ptiles || (qt - p.n_ptiles) < p.g.ff;
}

// Bounded wait by one thread.
__device__ __forceinline__ bool wait1(Smem& sm, const AttnParams& p, uint64_t* bar, uint32_t parity) {
  return rf_wait(bar, parity, &sm.abort, p.status, RF_ERR_TIMEOUT, p.wait_limit_ns);
}
// Bounded wait by a whole warp, with a warp-uniform outcome (the warp then
// runs .sync.aligned tcgen05 instructions together or leaves together).
__device__ __forceinline__ bool waitw(Smem& sm, const AttnParams& p, uint64_t* bar, uint32_t parity) {
  return __all_sync(0xFFFFFFFFu, wait1(sm, p, bar, parity));
}
// Parity of completion number n (0-based) of a barrier phase.
__device__ __forceinline__ uint32_t ph(uint32_t n) { return n & 1u; }

// Rendezvous of the two softmax warps that share a row quadrant, on an
// mbarrier (bounded wait, so a warp that leaves on an abort cannot strand its
// partner).  Orders each thread's earlier shared-memory writes before the
// partner's later reads.
__device__ __forceinline__ bool pair_sync(Smem& sm, const AttnParams& p, int quad, uint32_t& phase) {
  mbar_arrive(&sm.xbar[quad]);
  return waitw(sm, p, &sm.xbar[quad], ph(phase++));
}

// ---------------------------------------------------------------- producer
// Visits the KV tile rows of one unit in order: every prefix tile, then every
// sparse block (dense unit) or the set bits of its mask row.
struct KvIter {
  int base, n_ptiles, nb, words;
  const uint32_t* mrow;   // nullptr for a dense unit
  int t, wd;
  uint32_t bits;
  __device__ void init(int base_, const AttnParams& p, const uint32_t* mrow_) {
    base = base_;
    n_ptiles = p.n_ptiles;
    nb = p.g.nb;
    words = p.g.mask_words;
    mrow = mrow_;
    t = 0;
    wd = 0;
    bits = 0;
  }
  // Row of the next KV tile, or -1 at the end.
  __device__ int next() {
    if (t < n_ptiles) return base + (t++) * RF_BLOCK;
    if (!mrow) {
      const int j = t - n_ptiles;
      if (j >= nb) return -1;
      ++t;
      return base + (n_ptiles + j) * RF_BLOCK;
    }
    while (bits == 0) {
      if (wd >= words) return -1;
      bits = mrow[wd++];
    }
    const int j = 32 * (wd - 1) + __ffs(bits) - 1;
    bits &= bits - 1;
    return base + (n_ptiles + j) * RF_BLOCK;
  }
};

__device__ void producer_loop(Smem& sm, const AttnParams& p, const CUtensorMap* tq, const CUtensorMap* tk,
                              const CUtensorMap* tv) {
  const uint64_t pol_q = l2_policy_evict_first();
  const uint64_t pol_kv = l2_policy_evict_last();
  uint32_t c = 0, gk = 0, gv = 0;   // units, K tiles and V tiles issued
  const int S_int = p.g.S_int;
  bool ok = true;

  auto load_k = [&](int row) -> bool {
    const uint32_t st = gk % kKStages, use = gk / kKStages;
    if (use > 0 && !wait1(sm, p, &sm.k_empty[st], ph(use - 1))) return false;
    mbar_arrive_expect_tx(&sm.k_full[st], kTileBytes);
    tma_load_2d(sm.k[st], tk, &sm.k_full[st], 0, row, pol_kv);
    tma_load_2d(sm.k[st] + kHalfBytes, tk, &sm.k_full[st], 64, row, pol_kv);
    ++gk;
    return true;
  };
  auto load_v = [&](int row) -> bool {
    const uint32_t st = gv % kVStages, use = gv / kVStages;
    if (use > 0 && !wait1(sm, p, &sm.v_empty[st], ph(use - 1))) return false;
    mbar_arrive_expect_tx(&sm.v_full[st], kTileBytes);
    tma_load_2d(sm.v[st], tv, &sm.v_full[st], 0, row, pol_kv);
    tma_load_2d(sm.v[st] + kHalfBytes, tv, &sm.v_full[st], 64, row, pol_kv);
    ++gv;
    return true;
  };

  while (ok) {
    const int w = atomicAdd(p.counter, 1);
    const uint32_t slot = c & 1;
    if (c >= 2 && !wait1(sm, p, &sm.item_empty[slot], ph((c >> 1) - 1))) {
      ok = false;
      break;
    }
    Item itm{-1, 0, 0, 0};
    const uint32_t* mrow = nullptr;
    if (w < p.total_items) {
      itm.bn = w / p.g.n_tiles;
      itm.qt = w - itm.bn * p.g.n_tiles;
      if (is_dense_tile(p, itm.qt)) {
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
    if (itm.bn < 0) break;

    const int base = itm.bn * S_int;
    if (c >= 1 && !wait1(sm, p, &sm.q_empty, ph(c - 1))) {
      ok = false;
      break;
    }
    if (!(p.skip_first_q && c == 0)) {
      mbar_arrive_expect_tx(&sm.q_full, kTileBytes);
      tma_load_2d(sm.q, tq, &sm.q_full, 0, base + itm.qt * RF_BLOCK, pol_q);
      tma_load_2d(sm.q + kHalfBytes, tq, &sm.q_full, 64, base + itm.qt * RF_BLOCK, pol_q);
    }
    ++c;

    // K runs kKAhead tiles ahead of V: K0, K1, K2, V0, K3, V1, ..., V(n-1).
    KvIter kit, vit;
    kit.init(base, p, mrow);
    vit.init(base, p, mrow);
    for (int i = 0; i < kKAhead && ok; ++i) {
      const int rk = kit.next();
      if (rk < 0) break;
      ok = load_k(rk);
    }
    while (ok) {
      const int rk = kit.next();
      if (rk >= 0) ok = load_k(rk);
      if (!ok) break;
      const int rv = vit.next();
      if (rv < 0) break;
      ok = load_v(rv);
    }
  }
  if (!ok) {
    // Let the copies already issued land before the CTA may exit (bounded by
    // time, not cut short by the abort flag).
    const uint64_t lim = p.wait_limit_ns / 4;
    if (c) rf_wait_time(&sm.q_full, ph(c - 1), lim);
    for (uint32_t st = 0; st < kKStages; ++st) {
      const uint32_t nk = (gk > st) ? (gk - st + kKStages - 1) / kKStages : 0;
      if (nk) rf_wait_time(&sm.k_full[st], ph(nk - 1), lim);
    }
    for (uint32_t st = 0; st < kVStages; ++st) {
      const uint32_t nv = (gv > st) ? (gv - st + kVStages - 1) / kVStages : 0;
      if (nv) rf_wait_time(&sm.v_full[st], ph(nv - 1), lim);
    }
  }
}

// ---------------------------------------------------------------- MMA issuer
// Descriptor low words of the 128-byte swizzled operands; every descriptor
// used here shares one high word (stride 1024 B, sm_100 version, swizzle).
// A K step of 16 elements advances a K-major operand by 32 B (2 in the
// descriptor's 16-byte units), and the second 64-column half by 16 KB.
__device__ __forceinline__ void issue_qk(uint32_t s_tmem, uint32_t q_lo, uint32_t k_lo, uint32_t hi) {
  constexpr uint32_t idesc = make_idesc_bf16(128, 128, false);
#pragma unroll
  for (int kk = 0; kk < 8; ++kk) {
    const uint32_t off = ((kk >> 2) * kHalfBytes + (kk & 3) * 32) >> 4;
    mma_ss_lo(s_tmem, q_lo + off, k_lo + off, hi, idesc, kk > 0);
  }
}
// V is MN-major: a K step of 16 keys advances it by 16 rows of 128 B.
__device__ __forceinline__ void issue_pv(uint32_t o_tmem, uint32_t p_tmem, uint32_t v_lo, uint32_t hi,
                                         bool accumulate) {
  constexpr uint32_t idesc = make_idesc_bf16(128, 128, true);
#pragma unroll
  for (int kk = 0; kk < 8; ++kk)
    mma_ts_lo(o_tmem, p_tmem + kk * 8, v_lo + kk * (2048 >> 4), hi, idesc, (accumulate || kk > 0) ? 1u : 0u);
}

__device__ bool mma_loop_body(Smem& sm, const AttnParams& p, uint32_t tmem) {
  uint32_t c = 0, g = 0;   // units and KV tiles consumed
  const uint32_t hi = (uint32_t)(make_sdesc_sw128(0, 16, 1024) >> 32);
  const uint32_t q_lo = (uint32_t)make_sdesc_sw128(smem_u32(sm.q), 16, 1024);
  const uint32_t k_lo0 = (uint32_t)make_sdesc_sw128(smem_u32(sm.k[0]), 16, 1024);
  const uint32_t v_lo0 = (uint32_t)make_sdesc_sw128(smem_u32(sm.v[0]), kHalfBytes, 1024);
  // S of tile t into buffer t % 2: needs K tile t and S of tile t-2 read by the softmax.
  auto qk = [&](uint32_t t) -> bool {
    const uint32_t st = t % kKStages, sb = t & 1;
    if (!wait1(sm, p, &sm.k_full[st], ph(t / kKStages))) return false;
    if (t >= 2 && !wait1(sm, p, &sm.s_read[sb], ph((t >> 1) - 1))) return false;
    tc_fence_after();
    issue_qk(tmem + kColS + 128 * sb, q_lo, k_lo0 + st * (kTileBytes >> 4), hi);
    mma_commit(&sm.s_full[sb]);
    mma_commit(&sm.k_empty[st]);
    return true;
  };
  for (;;) {
    const uint32_t slot = c & 1;
    if (!wait1(sm, p, &sm.item_full[slot], ph(c >> 1))) return false;
    const Item itm = sm.items[slot];
    mbar_arrive(&sm.item_empty[slot]);
    if (itm.bn < 0) return true;
    const uint32_t n = itm.ntiles;
    if (!wait1(sm, p, &sm.q_full, ph(c))) return false;
    if (!qk(g)) return false;
    if (n == 1) mma_commit(&sm.q_empty);
    for (uint32_t j = 0; j < n; ++j) {
      const uint32_t t = g + j, pb = t & 1, vs = t % kVStages;
      if (j + 1 < n) {
        if (!qk(t + 1)) return false;
        if (j + 2 == n) mma_commit(&sm.q_empty);
      }
      if (!wait1(sm, p, &sm.p_full[pb], ph(t >> 1))) return false;
      if (!wait1(sm, p, &sm.v_full[vs], ph(t / kVStages))) return false;
      // the epilogue of the previous unit must have read O
      if (j == 0 && c >= 1 && !wait1(sm, p, &sm.o_empty, ph(c - 1))) return false;
      tc_fence_after();
      issue_pv(tmem + kColO, tmem + kColP + 64 * pb, v_lo0 + vs * (kTileBytes >> 4), hi, j > 0);
      mma_commit(&sm.p_free[pb]);
      mma_commit(&sm.v_empty[vs]);
      if (j + 1 == n) mma_commit(&sm.o_full);
    }
    g += n;
    ++c;
  }
}

// Leaves after the last unit, or early on an abort; in the latter case the
// MMAs already issued must finish before tensor memory is freed.
__device__ void mma_loop(Smem& sm, const AttnParams& p, uint32_t tmem) {
  if (!mma_loop_body(sm, p, tmem)) {
    mma_commit(&sm.drain);
    rf_wait_time(&sm.drain, 0, p.wait_limit_ns / 4);
  }
}

// ---------------------------------------------------------------- softmax + epilogue
__device__ void softmax_loop(Smem& sm, const AttnParams& p, uint32_t tmem) {
  const int warp = threadIdx.x >> 5;           // 0..7
  const int quad = warp & 3, half = warp >> 2;
  const int row = quad * 32 + (threadIdx.x & 31);   // query row == TMEM lane
  const uint32_t lane_base = tmem + ((uint32_t)(quad * 32) << 16);
  const uint32_t tO = lane_base + kColO + 64 * half;
  const int col0 = 64 * half;                  // first key column of this thread
  const float sl2 = p.scale_log2;
  const uint64_t sl2x2 = f2_pack(sl2, sl2);
  uint32_t c = 0, g = 0, xph = 0;
  for (;;) {
    const uint32_t slot = c & 1;
    if (!waitw(sm, p, &sm.item_full[slot], ph(c >> 1))) return;
    const Item itm = sm.items[slot];
    mbar_arrive(&sm.item_empty[slot]);
    if (itm.bn < 0) return;

    float m_use = -CUDART_INF_F, l = 0.f;
    for (int j = 0; j < itm.ntiles; ++j) {
      const uint32_t t = g + j, sb = t & 1;
      const uint32_t tS = lane_base + kColS + 128 * sb + col0;
      const uint32_t tP = lane_base + kColP + 64 * sb + 32 * half;
      if (!waitw(sm, p, &sm.s_full[sb], ph(t >> 1))) return;
      tc_fence_after();
      uint32_t s[2][32];
      tmem_ld32(tS, s[0]);
      tmem_ld32(tS + 32, s[1]);
      tmem_wait_ld();
      reg_fence32(s[0]);
      reg_fence32(s[1]);
      // S is in registers: the tensor pipe may overwrite this buffer.
      tc_fence_before();
      mbar_arrive(&sm.s_read[sb]);

      const bool partial = (p.p_rem != 0 && j == p.n_ptiles - 1);
      if (partial) {
#pragma unroll
        for (int q2 = 0; q2 < 2; ++q2)
#pragma unroll
          for (int e = 0; e < 32; ++e)
            if (col0 + 32 * q2 + e >= p.p_rem) s[q2][e] = __float_as_uint(-CUDART_INF_F);
      }
      // row max over this half: 8 independent chains of 3-input max
      float mx8[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) mx8[i] = -CUDART_INF_F;
#pragma unroll
      for (int q2 = 0; q2 < 2; ++q2)
#pragma unroll
        for (int e = 0; e < 32; e += 2)
          mx8[(e >> 1) & 7] = max3f(mx8[(e >> 1) & 7], __uint_as_float(s[q2][e]), __uint_as_float(s[q2][e + 1]));
      const float mxh = max3f(max3f(mx8[0], mx8[1], mx8[2]), max3f(mx8[3], mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7]));
      // combine with the other half of the row
      sm.xmax[sb][half][row] = mxh;
      if (!pair_sync(sm, p, quad, xph)) return;
      const float mx = fmaxf(mxh, sm.xmax[sb][half ^ 1][row]);
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
      // p = 2^(s * scale * log2 e - m): pairs, packed fp32 arithmetic
      const uint64_t negm = f2_pack(-m_use, -m_use);
      uint64_t sum2[4] = {0, 0, 0, 0};
      uint32_t pk[32];
#pragma unroll
      for (int q2 = 0; q2 < 2; ++q2)
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          const int i = 16 * q2 + (e >> 1);     // pair index 0..31 within this half
          const uint64_t x2 = f2_fma(f2_pack(__uint_as_float(s[q2][e]), __uint_as_float(s[q2][e + 1])), sl2x2, negm);
          uint64_t p2;
          if ((i % kPolyEvery) == kPolyEvery - 1) {
            p2 = exp2_poly_x2(x2);
          } else {
            float x0, x1;
            f2_unpack(x2, x0, x1);
            p2 = f2_pack(ex2_approx(x0), ex2_approx(x1));
          }
          if (partial) {
            float a0, a1;
            f2_unpack(p2, a0, a1);
            const int k0 = col0 + 2 * i;
            p2 = f2_pack(k0 < p.p_rem ? a0 : 0.f, k0 + 1 < p.p_rem ? a1 : 0.f);
          }
          sum2[i & 3] = f2_add(sum2[i & 3], p2);
          float a0, a1;
          f2_unpack(p2, a0, a1);
          pk[i] = pack_bf16x2(a0, a1);
        }
      float s0, s1, s2, s3;
      f2_unpack(f2_add(sum2[0], sum2[1]), s0, s1);
      f2_unpack(f2_add(sum2[2], sum2[3]), s2, s3);
      l = l * alpha + ((s0 + s1) + (s2 + s3));
      if (__any_sync(0xFFFFFFFFu, rescale)) {
        // O holds the tiles before j once the P*V of tile j-1 is done.
        if (!waitw(sm, p, &sm.p_free[(t - 1) & 1], ph((t - 1) >> 1))) return;
        tc_fence_after();
#pragma unroll 1
        for (int q2 = 0; q2 < 2; ++q2) {
          uint32_t o[32];
          tmem_ld32(tO + 32 * q2, o);
          tmem_wait_ld();
          reg_fence32(o);
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
          tmem_st32(tO + 32 * q2, o);
        }
      }
      // P buffer sb is free once the P*V of tile t-2 is done
      if (t >= 2 && !waitw(sm, p, &sm.p_free[sb], ph((t >> 1) - 1))) return;
      tc_fence_after();
      tmem_st32(tP, pk);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&sm.p_full[sb]);
    }
    // epilogue: O / l of this unit once its last P*V is done
    if (!waitw(sm, p, &sm.o_full, ph(c))) return;
    tc_fence_after();
    uint32_t o[2][32];
    tmem_ld32(tO, o[0]);
    tmem_ld32(tO + 32, o[1]);
    tmem_wait_ld();
    reg_fence32(o[0]);
    reg_fence32(o[1]);
    // O is in registers: the next unit may start accumulating.
    tc_fence_before();
    mbar_arrive(&sm.o_empty);
    // xsum is rewritten only at the end of the next unit, after at least one
    // more rendezvous, so one rendezvous here is enough.
    sm.xsum[half][row] = l;
    if (!pair_sync(sm, p, quad, xph)) return;
    const float rl = 1.f / (sm.xsum[0][row] + sm.xsum[1][row]);
    const int b = itm.bn / p.N, n = itm.bn - b * p.N;
    const int src = rf_src_of_row(p.g, itm.qt * RF_BLOCK + row);
    if (src >= 0) {
      __nv_bfloat16* dst = p.out + rf_token_offset(p.layout, p.B, p.S, p.N, b, n, src) + col0;
#pragma unroll
      for (int q2 = 0; q2 < 2; ++q2) {
        uint32_t w[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
          w[e] = pack_bf16x2(__uint_as_float(o[q2][2 * e]) * rl, __uint_as_float(o[q2][2 * e + 1]) * rl);
        uint4* d4 = reinterpret_cast<uint4*>(dst + 32 * q2);
#pragma unroll
        for (int e = 0; e < 4; ++e) d4[e] = make_uint4(w[4 * e], w[4 * e + 1], w[4 * e + 2], w[4 * e + 3]);
      }
    }
    g += itm.ntiles;
    ++c;
  }
}

__global__ void __launch_bounds__(kThreads, 1)
    attn_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const AttnParams p) {
  extern __shared__ uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(&sm.q_full, 1);
    mbar_init(&sm.q_empty, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sm.s_full[i], 1);
      mbar_init(&sm.s_read[i], kSoftmaxThreads);
      mbar_init(&sm.p_full[i], kSoftmaxThreads);
      mbar_init(&sm.p_free[i], 1);
      mbar_init(&sm.item_full[i], 1);
      mbar_init(&sm.item_empty[i], kSoftmaxThreads + 1);
    }
    for (int i = 0; i < kKStages; ++i) {
      mbar_init(&sm.k_full[i], 1);
      mbar_init(&sm.k_empty[i], 1);
    }
    for (int i = 0; i < kVStages; ++i) {
      mbar_init(&sm.v_full[i], 1);
      mbar_init(&sm.v_empty[i], 1);
    }
    mbar_init(&sm.o_full, 1);
    mbar_init(&sm.drain, 1);
    mbar_init(&sm.o_empty, kSoftmaxThreads);
    for (int i = 0; i < 4; ++i) mbar_init(&sm.xbar[i], 64);
    sm.abort = 0;
    fence_mbar_init();
  }
  if (warp == 8 && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  if (warp == 9) {
    tmem_alloc(&sm.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;

  if (warp < 8) {
    softmax_loop(sm, p, tmem);
  } else if (warp == 8) {
    if (lane == 0) producer_loop(sm, p, &tm_q, &tm_k, &tm_v);
  } else {
    if (lane == 0) mma_loop(sm, p, tmem);
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 9) tmem_dealloc(tmem, kTmemCols);
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
                             int* counter, int* status, const AttnDebug& dbg, cudaStream_t stream) {
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
  p.wait_limit_ns = dbg.wait_limit_ns > 0 ? (uint64_t)dbg.wait_limit_ns : kWaitLimitNs;
  p.skip_first_q = dbg.skip_first_q;

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
  const int grid = std::min(sms, p.total_items);
  attn_kernel<<<grid, kThreads, smem, stream>>>(tq, tk, tv, p);
  return cudaGetLastError();
}

}  // namespace rf
