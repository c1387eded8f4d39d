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
// A CTA runs two units at once in two independent slots, each with its own
// Q/K/V shared-memory buffers, its own S and O in tensor memory and its own
// warps, so that while the softmax of one slot runs the tensor pipe works on
// the other slot's MMAs:
//   warps 0-3   slot 0, warps 4-7 slot 1: thread = query row (TMEM lane);
//               online softmax in exp2 with a lazily updated running max;
//               most exponentials on the MUFU unit, one pair in four on the
//               FMA pipe (polynomial); P (bf16) is written over the first 64
//               columns of the slot's S; at the end of a unit the same
//               threads write O / l -> bf16 -> the caller's layout.  The
//               slot's first warp also issues its MMAs (one elected lane):
//               S = Q K^T: tcgen05 kind::f16, A and B from shared memory;
//               O += P V:  A = P from tensor memory, B = V MN-major.
//               The four warps meet at a named barrier after each tile, so
//               P V follows P without an mbarrier hand-off.
//   warps 8, 9  TMA producers of slot 0 and slot 1 (one thread each): Q, then
//               the K and V tiles of the KV list, 128-byte swizzled boxes of
//               128 rows x 64 columns.
//   warp 10     owns the tensor memory; warps 10 and 11 are otherwise idle.
// Tensor memory (512 columns): slot z has S at [256 z, 256 z + 128) (P in
// its first 64 columns) and O at [256 z + 128, 256 z + 256).  Since P
// overwrites S, the QK of a slot's next tile is issued once its P V is done.
// Registers: the control warpgroup (warps 8-11) gives registers to the two
// slot warpgroups (setmaxnreg 64 / 216: 8 x 32 x 216 + 4 x 32 x 64 =
// 63,488 <= 384 threads x 168 at launch).
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

constexpr int kThreads = 384;
constexpr int kSlots = 2;
constexpr int kSlotWarps = 4;                            // softmax warps per slot
constexpr uint32_t kRegsSoftmax = 216, kRegsControl = 64;
constexpr int kTileBytes = RF_BLOCK * RF_HEAD_DIM * 2;   // 32 KB
constexpr int kHalfBytes = kTileBytes / 2;               // 64 columns x 128 rows
constexpr uint32_t kTmemCols = 512;
constexpr int kPolyEvery = 4;                            // pair i uses the polynomial when i % 4 == 3
constexpr float kRescaleThreshold = 8.0f;                // log2 units
constexpr uint64_t kWaitLimitNs = 2000000000ull;

struct Item {
  int bn, qt, ntiles, pad;
};

// One slot: buffers and barriers of one unit in flight.
struct __align__(1024) Slot {
  uint8_t q[kTileBytes];
  uint8_t k[kTileBytes];
  uint8_t v[kTileBytes];
  uint64_t q_full, q_empty, k_full, k_empty, v_full, v_empty;
  uint64_t s_full, pv_done;
  uint64_t drain;               // the issuer's last commit when it leaves early
  uint64_t item_full[2], item_empty[2];
  Item items[2];
};

struct Smem {
  Slot slot[kSlots];
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
// One arrival per warp, after every lane's preceding work (callers fence first).
__device__ __forceinline__ void arrive_w(uint64_t* bar) {
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(bar);
}
// Parity of completion number n (0-based) of a barrier phase.
__device__ __forceinline__ uint32_t ph(uint32_t n) { return n & 1u; }

template <uint32_t N>
__device__ __forceinline__ void regs_increase() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}
template <uint32_t N>
__device__ __forceinline__ void regs_decrease() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
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

// Producer of one slot: takes units from the global counter, loads Q and then
// the K and V tiles of the KV list (one buffer each; K of the next tile as
// soon as the previous S = Q K^T is done, V as soon as the previous P V is).
__device__ void producer_loop(Smem& sm, Slot& sl, const AttnParams& p, const CUtensorMap* tq, const CUtensorMap* tk,
                              const CUtensorMap* tv) {
  const uint64_t pol_q = l2_policy_evict_first();
  const uint64_t pol_kv = l2_policy_evict_last();
  uint32_t c = 0, nk = 0, nv = 0;   // units, K tiles and V tiles issued
  const int S_int = p.g.S_int;
  bool ok = true;
  while (ok) {
    const int w = atomicAdd(p.counter, 1);
    const uint32_t it = c & 1;
    if (c >= 2 && !wait1(sm, p, &sl.item_empty[it], ph((c >> 1) - 1))) {
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
    sl.items[it] = itm;
    mbar_arrive(&sl.item_full[it]);
    if (itm.bn < 0) break;

    const int base = itm.bn * S_int;
    if (c >= 1 && !wait1(sm, p, &sl.q_empty, ph(c - 1))) {
      ok = false;
      break;
    }
    if (!(p.skip_first_q && c == 0)) {
      mbar_arrive_expect_tx(&sl.q_full, kTileBytes);
      tma_load_2d(sl.q, tq, &sl.q_full, 0, base + itm.qt * RF_BLOCK, pol_q);
      tma_load_2d(sl.q + kHalfBytes, tq, &sl.q_full, 64, base + itm.qt * RF_BLOCK, pol_q);
    }
    ++c;
    KvIter kit;
    kit.init(base, p, mrow);
    for (int row = kit.next(); row >= 0 && ok; row = kit.next()) {
      if (nk >= 1 && !wait1(sm, p, &sl.k_empty, ph(nk - 1))) {
        ok = false;
        break;
      }
      mbar_arrive_expect_tx(&sl.k_full, kTileBytes);
      tma_load_2d(sl.k, tk, &sl.k_full, 0, row, pol_kv);
      tma_load_2d(sl.k + kHalfBytes, tk, &sl.k_full, 64, row, pol_kv);
      ++nk;
      if (nv >= 1 && !wait1(sm, p, &sl.v_empty, ph(nv - 1))) {
        ok = false;
        break;
      }
      mbar_arrive_expect_tx(&sl.v_full, kTileBytes);
      tma_load_2d(sl.v, tv, &sl.v_full, 0, row, pol_kv);
      tma_load_2d(sl.v + kHalfBytes, tv, &sl.v_full, 64, row, pol_kv);
      ++nv;
    }
  }
  if (!ok) {
    // Let the copies already issued land before the CTA may exit (bounded by
    // time, not cut short by the abort flag).
    const uint64_t lim = p.wait_limit_ns / 4;
    if (c) rf_wait_time(&sl.q_full, ph(c - 1), lim);
    if (nk) rf_wait_time(&sl.k_full, ph(nk - 1), lim);
    if (nv) rf_wait_time(&sl.v_full, ph(nv - 1), lim);
  }
}

// ---------------------------------------------------------------- MMA issue
// Descriptor low words of the 128-byte swizzled operands; every descriptor
// used here shares one high word (stride 1024 B, sm_100 version, swizzle).
// A K step of 16 elements advances a K-major operand by 32 B (2 in the
// descriptor's 16-byte units), and the second 64-column half by 16 KB.
// The issuing warp runs this code together; one elected lane issues.
__device__ __forceinline__ void issue_qk(uint32_t s_tmem, uint32_t q_lo, uint32_t k_lo, uint32_t hi) {
  constexpr uint32_t idesc = make_idesc_bf16(128, 128, false);
#pragma unroll
  for (int kk = 0; kk < 8; ++kk) {
    const uint32_t off = ((kk >> 2) * kHalfBytes + (kk & 3) * 32) >> 4;
    mma_ss_lo_elect(s_tmem, q_lo + off, k_lo + off, hi, idesc, kk > 0);
  }
}
// V is MN-major: a K step of 16 keys advances it by 16 rows of 128 B.
__device__ __forceinline__ void issue_pv(uint32_t o_tmem, uint32_t p_tmem, uint32_t v_lo, uint32_t hi,
                                         bool accumulate) {
  constexpr uint32_t idesc = make_idesc_bf16(128, 128, true);
#pragma unroll
  for (int kk = 0; kk < 8; ++kk)
    mma_ts_lo_elect(o_tmem, p_tmem + kk * 8, v_lo + kk * (2048 >> 4), hi, idesc, (accumulate || kk > 0) ? 1u : 0u);
}

// Rendezvous of a slot's four warps (named barrier `id`, 128 threads) that
// also returns whether every thread passed `ok`: the warps of a slot leave
// together, so none is left waiting at a later rendezvous.
__device__ __forceinline__ bool slot_vote(int id, bool ok) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred a, b;\n\tsetp.ne.u32 a, %1, 0;\n\t"
      "bar.red.and.pred b, %2, 128, a;\n\tselp.u32 %0, 1, 0, b;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)ok), "r"(id)
      : "memory");
  return r != 0;
}

// ---------------------------------------------------------------- softmax of one tile
// Thread = query row.  Reads the row's 128 scores from S, updates the running
// max m_use (log2 units, lazily: only when a score exceeds it by more than
// the threshold, then O and l are rescaled), adds the tile's sum to l and
// writes P = 2^(s * scale * log2 e - m_use) as bf16 over the first 64
// columns of S.  `p_valid` < 128 masks the keys past the prefix's end.
__device__ __forceinline__ void softmax_tile(uint32_t tS, uint32_t tO, bool first, int p_valid, float sl2,
                                             float& m_use, float& l) {
  const uint64_t sl2x2 = f2_pack(sl2, sl2);
  uint32_t s[4][32];
#pragma unroll
  for (int q4 = 0; q4 < 4; ++q4) tmem_ld32(tS + 32 * q4, s[q4]);
  tmem_wait_ld();
#pragma unroll
  for (int q4 = 0; q4 < 4; ++q4) reg_fence32(s[q4]);

  const bool partial = p_valid < RF_BLOCK;
  if (partial) {
#pragma unroll
    for (int q4 = 0; q4 < 4; ++q4)
#pragma unroll
      for (int e = 0; e < 32; ++e)
        if (32 * q4 + e >= p_valid) s[q4][e] = __float_as_uint(-CUDART_INF_F);
  }
  float mx8[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) mx8[i] = -CUDART_INF_F;
#pragma unroll
  for (int q4 = 0; q4 < 4; ++q4)
#pragma unroll
    for (int e = 0; e < 32; e += 2)
      mx8[(e >> 1) & 7] = max3f(mx8[(e >> 1) & 7], __uint_as_float(s[q4][e]), __uint_as_float(s[q4][e + 1]));
  const float mx = max3f(max3f(mx8[0], mx8[1], mx8[2]), max3f(mx8[3], mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7]));
  const float mx_s = mx * sl2;
  float alpha = 1.f;
  bool rescale = false;
  if (first) {
    m_use = mx_s;
  } else if (mx_s > m_use + kRescaleThreshold) {
    alpha = ex2_approx(m_use - mx_s);
    m_use = mx_s;
    rescale = true;
  }
  const uint64_t negm = f2_pack(-m_use, -m_use);
  uint64_t sum2[4] = {0, 0, 0, 0};
  uint32_t pk[64];
#pragma unroll
  for (int q4 = 0; q4 < 4; ++q4)
#pragma unroll
    for (int e = 0; e < 32; e += 2) {
      const int i = 16 * q4 + (e >> 1);     // pair index 0..63
      const uint64_t x2 = f2_fma(f2_pack(__uint_as_float(s[q4][e]), __uint_as_float(s[q4][e + 1])), sl2x2, negm);
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
        p2 = f2_pack(2 * i < p_valid ? a0 : 0.f, 2 * i + 1 < p_valid ? a1 : 0.f);
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
    // O holds the tiles before this one: their P V completed before this
    // tile's S = Q K^T was issued.
#pragma unroll 1
    for (int q4 = 0; q4 < 4; ++q4) {
      uint32_t o[32];
      tmem_ld32(tO + 32 * q4, o);
      tmem_wait_ld();
      reg_fence32(o);
#pragma unroll
      for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
      tmem_st32(tO + 32 * q4, o);
    }
  }
  tmem_st32(tS, *reinterpret_cast<uint32_t(*)[32]>(&pk[0]));
  tmem_st32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&pk[32]));
  tmem_wait_st();
  tc_fence_before();
}

// ---------------------------------------------------------------- one slot
// The slot's four warps compute the softmax of each tile (thread = query row
// = TMEM lane) and write the unit's output; the first of them also issues
// the slot's MMAs: S = Q K^T of a tile once the P V of the previous tile is
// done (P lives in the S columns), and P V of a tile once all four warps
// have written P (the rendezvous after each tile).
__device__ void slot_loop(Smem& sm, Slot& sl, const AttnParams& p, uint32_t tmem_slot, int bar_id) {
  const int quad = (threadIdx.x >> 5) & 3;
  const bool issuer = (quad == 0);
  const int row = quad * 32 + (threadIdx.x & 31);   // query row == TMEM lane
  const uint32_t lane_base = tmem_slot + ((uint32_t)(quad * 32) << 16);
  const uint32_t tS = lane_base, tO = lane_base + 128;
  const uint32_t s_tmem = tmem_slot, o_tmem = tmem_slot + 128;
  const uint32_t hi = (uint32_t)(make_sdesc_sw128(0, 16, 1024) >> 32);
  const uint32_t q_lo = (uint32_t)make_sdesc_sw128(smem_u32(sl.q), 16, 1024);
  const uint32_t k_lo = (uint32_t)make_sdesc_sw128(smem_u32(sl.k), 16, 1024);
  const uint32_t v_lo = (uint32_t)make_sdesc_sw128(smem_u32(sl.v), kHalfBytes, 1024);
  uint32_t c = 0, t = 0;   // units and tiles of this slot
  bool ok = true;
  bool issued = false;     // the issuer has MMAs that may still run

  // S = Q K^T of tile t (issuer warp): K tile t must have landed and the
  // P V of tile t-1 must be done.
  auto qk = [&](uint32_t tt, bool last_of_unit) -> bool {
    if (!waitw(sm, p, &sl.k_full, ph(tt))) return false;
    if (tt >= 1 && !waitw(sm, p, &sl.pv_done, ph(tt - 1))) return false;
    tc_fence_after();
    issue_qk(s_tmem, q_lo, k_lo, hi);
    mma_commit_elect(&sl.s_full);
    mma_commit_elect(&sl.k_empty);
    if (last_of_unit) mma_commit_elect(&sl.q_empty);
    issued = true;
    return true;
  };

  for (;; ++c) {
    // Every warp of the slot reaches every rendezvous: a warp whose wait
    // failed carries ok = false to the next one, where all four leave.
    const uint32_t it = c & 1;
    Item itm{-1, 0, 0, 0};
    if (ok) ok = waitw(sm, p, &sl.item_full[it], ph(c >> 1));
    if (ok) {
      itm = sl.items[it];
      arrive_w(&sl.item_empty[it]);
    }
    ok = slot_vote(bar_id, ok);
    if (!ok || itm.bn < 0) break;
    if (issuer) ok = waitw(sm, p, &sl.q_full, ph(c)) && qk(t, itm.ntiles == 1);

    float m_use = -CUDART_INF_F, l = 0.f;
    for (int j = 0; j < itm.ntiles; ++j, ++t) {
      if (ok) ok = waitw(sm, p, &sl.s_full, ph(t));
      if (ok) {
        tc_fence_after();
        const int p_valid = (p.p_rem != 0 && j == p.n_ptiles - 1) ? p.p_rem : RF_BLOCK;
        softmax_tile(tS, tO, j == 0, p_valid, p.scale_log2, m_use, l);
      }
      ok = slot_vote(bar_id, ok);
      if (!ok) break;
      if (issuer) {
        ok = waitw(sm, p, &sl.v_full, ph(t));
        if (ok) {
          tc_fence_after();
          issue_pv(o_tmem, s_tmem, v_lo, hi, j > 0);
          mma_commit_elect(&sl.pv_done);
          mma_commit_elect(&sl.v_empty);
          if (j + 1 < itm.ntiles) ok = qk(t + 1, j + 2 == itm.ntiles);
        }
      }
    }
    // epilogue: O / l of this unit once its last P V is done
    if (ok) ok = waitw(sm, p, &sl.pv_done, ph(t - 1));
    if (ok) {
      tc_fence_after();
      const float rl = 1.f / l;
      const int b = itm.bn / p.N, nh = itm.bn - b * p.N;
      const int src = rf_src_of_row(p.g, itm.qt * RF_BLOCK + row);
      __nv_bfloat16* dst = src >= 0 ? p.out + rf_token_offset(p.layout, p.B, p.S, p.N, b, nh, src) : nullptr;
#pragma unroll 1
      for (int q4 = 0; q4 < 4; ++q4) {
        uint32_t o[32];
        tmem_ld32(tO + 32 * q4, o);
        tmem_wait_ld();
        reg_fence32(o);
        if (dst) {
          uint32_t w[16];
#pragma unroll
          for (int e = 0; e < 16; ++e)
            w[e] = pack_bf16x2(__uint_as_float(o[2 * e]) * rl, __uint_as_float(o[2 * e + 1]) * rl);
          uint4* d4 = reinterpret_cast<uint4*>(dst + 32 * q4);
#pragma unroll
          for (int e = 0; e < 4; ++e) d4[e] = make_uint4(w[4 * e], w[4 * e + 1], w[4 * e + 2], w[4 * e + 3]);
        }
      }
      // The next unit's first P V overwrites O only after the rendezvous
      // that follows its first softmax tile, which ends with this fence.
      tc_fence_before();
    }
  }
  // Leaving early on an abort: the MMAs already issued must finish before
  // tensor memory is freed.
  if (!ok && issuer && issued) {
    mma_commit_elect(&sl.drain);
    rf_wait_time(&sl.drain, 0, p.wait_limit_ns / 4);
    __syncwarp();
  }
}

__global__ void __launch_bounds__(kThreads, 1)
    attn_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const AttnParams p) {
  extern __shared__ uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int z = 0; z < kSlots; ++z) {
      Slot& sl = sm.slot[z];
      mbar_init(&sl.q_full, 1);
      mbar_init(&sl.q_empty, 1);
      mbar_init(&sl.k_full, 1);
      mbar_init(&sl.k_empty, 1);
      mbar_init(&sl.v_full, 1);
      mbar_init(&sl.v_empty, 1);
      mbar_init(&sl.s_full, 1);
      mbar_init(&sl.pv_done, 1);
      mbar_init(&sl.drain, 1);
      for (int i = 0; i < 2; ++i) {
        mbar_init(&sl.item_full[i], 1);
        mbar_init(&sl.item_empty[i], kSlotWarps);
      }
    }
    sm.abort = 0;
    fence_mbar_init();
  }
  if (warp == 8 && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  if (warp == 10) {
    tmem_alloc(&sm.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;

  if (warp < 8) {
    regs_increase<kRegsSoftmax>();
    const int z = warp >> 2;
    slot_loop(sm, sm.slot[z], p, tmem + 256 * z, 1 + z);
  } else {
    regs_decrease<kRegsControl>();
    if (warp == 8 && lane == 0) producer_loop(sm, sm.slot[0], p, &tm_q, &tm_k, &tm_v);
    if (warp == 9 && lane == 0) producer_loop(sm, sm.slot[1], p, &tm_q, &tm_k, &tm_v);
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 10) tmem_dealloc(tmem, kTmemCols);
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
