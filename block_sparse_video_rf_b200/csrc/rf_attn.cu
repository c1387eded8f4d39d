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
// key prefix tile, then either every key block (dense tile) or the blocks
// set in its mask row, in ascending order.  Keys and values may have a
// geometry of their own (lite_boost.ops.sparse_attention, latent_shape_k):
// query tiles follow the query plan, KV tiles the key plan.  Persistent CTAs (one per SM) take
// units from a global counter in (head, tile) order, dense tiles of a head
// first, so the heads in flight keep their K/V in L2.
//
// A CTA runs two units at once in two independent slots, each with its own
// Q/K/V shared-memory buffers, its own S and O in tensor memory and its own
// warps, so that while the softmax of one slot runs the tensor pipe works on
// the other slot's MMAs:
//   warps 0-3   slot 0, warps 4-7 slot 1: thread = query row (TMEM lane);
//               online softmax in exp2 with a lazily updated running max
//               (a tile computes its own maximum only when its P would
//               exceed the format's range); most exponentials on the MUFU
//               unit, one pair in four (fp8: three) on the FMA pipe
//               (polynomial); P is written over the first columns of
//               the slot's S; at the end of a unit the same threads write
//               O / l in the caller's type and layout.  The slot's first warp
//               also issues its MMAs (one elected lane):
//                 S = Q K^T:  A and B from shared memory;
//                 O += P V:   A = P from tensor memory, B = V.
//               The four warps meet at a named barrier after each tile, so
//               P V follows P without an mbarrier hand-off.
//   warps 8, 9  TMA producers of slot 0 and slot 1 (one thread each): Q, then
//               the K and V tiles of the KV list, 128-byte swizzled boxes of
//               128 rows x 128 bytes.
//   warp 10     owns the tensor memory; warps 10 and 11 are otherwise idle.
// Tensor memory (512 columns): slot z has S at [256 z, 256 z + 128) (P in
// its first columns) and O at [256 z + 128, 256 z + 256).  Since P
// overwrites S, the QK of a slot's next tile is issued once its P V is done.
// Registers: the control warpgroup (warps 8-11) gives registers to the two
// slot warpgroups (setmaxnreg 64 / 216: 8 x 32 x 216 + 4 x 32 x 64 =
// 63,488 <= 384 threads x 168 at launch).
//
// Precisions (template parameters):
//   16-bit: Q, K, V and out bf16 or fp16; tcgen05 kind::f16, 8 MMAs of
//     128x128x16 per product; P in the input type (64 TMEM columns);
//     V MN-major; single K and V buffers per slot.
//   fp8: Q, K, V as e4m3 codes with one fp32 scale per 128-row block
//     (written by the quantisation kernel; V's blocks stored transposed so
//     that P V has a K-major B); tcgen05 kind::f8f6f4, 4 MMAs of 128x128x32
//     per product; S is scaled by sq * sk in the softmax; P is e4m3 (32 TMEM
//     columns) and carries the V block's scale relative to the head's
//     largest one (sv / vmax, folded into the exponent), which the epilogue
//     multiplies back; two K and two V buffers per slot.
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
constexpr int kBoxBytes = RF_BLOCK * 128;                // one TMA box: 128 rows x 128 bytes
constexpr uint32_t kTmemCols = 512;

constexpr float kRescaleThreshold = 8.0f;                // log2 units
constexpr uint64_t kWaitLimitNs = 2000000000ull;

// Compile-time shape of one precision.
template <bool kF16_, bool kFp8_>
struct Cfg {
  static constexpr bool kF16 = kF16_;                    // 16-bit type: fp16 (else bf16); also the output type
  static constexpr bool kFp8 = kFp8_;
  static constexpr int kBoxes = kFp8 ? 1 : 2;            // boxes per 128 x 128 tile
  static constexpr int kTileBytes = kBoxes * kBoxBytes;
  static constexpr int kKStages = kFp8 ? 2 : 1;
  static constexpr int kVStages = kFp8 ? 2 : 1;
  static constexpr int kSteps = kFp8 ? 4 : 8;            // MMAs per product over 128 (K 32 or 16 each)
  static constexpr int kPCols = kFp8 ? 32 : 64;          // TMEM columns of P
  // exponent pair i runs the polynomial on the FMA pipe when i % kPolyEvery == kPolyEvery - 1
  // (the rest on MUFU): measured best split for each path
  static constexpr int kPolyEvery = kFp8 ? 3 : 4;
  static constexpr uint32_t kIdescQK =
      kFp8 ? make_idesc_e4m3(128, 128, false) : make_idesc_f16kind(128, 128, false, !kF16);
  static constexpr uint32_t kIdescPV =
      kFp8 ? make_idesc_e4m3(128, 128, false) : make_idesc_f16kind(128, 128, true, !kF16);
};

struct Item {
  int bn, qt, ntiles, pad;
};

// Per-tile factors of the fp8 path, written by the slot's issuer before its
// arrival on s_full: c = scale * log2(e) * sq * sk (multiplies S), lr =
// log2(sv / vmax) (added to P's exponent), ir = vmax / sv (l adds P's sum
// times ir).
struct TileScale {
  float c, lr, ir, pad;
};

// One slot: buffers and barriers of one unit in flight.
template <class C>
struct __align__(1024) Slot {
  uint8_t q[C::kTileBytes];
  uint8_t k[C::kKStages][C::kTileBytes];
  uint8_t v[C::kVStages][C::kTileBytes];
  uint64_t q_full, q_empty;
  uint64_t k_full[C::kKStages], k_empty[C::kKStages], v_full[C::kVStages], v_empty[C::kVStages];
  uint64_t s_full;              // S = Q K^T of a tile done (commit) and its TileScale written (issuer)
  uint64_t pv_done;
  uint64_t drain;               // the issuer's last commit when it leaves early
  uint64_t item_full[2], item_empty[2];
  Item items[2];
  float q_scale;                // fp8: the unit's Q block scale (producer, with q_full)
  float kv_scale[C::kKStages][2];   // fp8: {sk, sv} of the tile in each K stage (producer, with k_full)
  TileScale ts[2];              // fp8: by tile parity (issuer, with s_full)
};

template <class C>
struct Smem {
  Slot<C> slot[kSlots];
  uint32_t tmem_base;
  int abort;
};

struct AttnParams {
  rf_plan_t g;       // query geometry (units, dense rows, the output's token order)
  rf_plan_t gk;      // key/value geometry (KV lists; the same as g unless k and v have their own)
  int B, S, N, layout;   // S: query sequence length (the output's)
  int total_items;
  int n_ptiles;      // query prefix tiles (g.P_pad / 128)
  int n_ptiles_k;    // key prefix tiles (gk.P_pad / 128)
  int p_rem_k;       // valid rows of the last key prefix tile when it is partial, else 0
  float scale_log2;
  const uint32_t* mask;  // [B*N, g.nb, gk.mask_words]
  const float* scales;   // fp8: q [B*N, g.n_tiles], then k and v [B*N, gk.n_tiles] block scales
  const float* vmax;     // fp8: [B*N] largest V block scale of each head
  int* counter;
  int* status;
  void* out;
  uint64_t wait_limit_ns;   // limit of every device-side wait
  int skip_first_q;         // test control: the first unit's Q load is never issued
};

__device__ __forceinline__ bool is_dense_tile(const AttnParams& p, int qt) {
  return p.g.dense || qt < p.n_ptiles || (qt - p.n_ptiles) < p.g.ff;
}

// Bounded wait by one thread.
template <class C>
__device__ __forceinline__ bool wait1(Smem<C>& sm, const AttnParams& p, uint64_t* bar, uint32_t parity) {
  return rf_wait(bar, parity, &sm.abort, p.status, RF_ERR_TIMEOUT, p.wait_limit_ns);
}
// Bounded wait by a whole warp, with a warp-uniform outcome (the warp then
// runs .sync.aligned tcgen05 instructions together or leaves together).
template <class C>
__device__ __forceinline__ bool waitw(Smem<C>& sm, const AttnParams& p, uint64_t* bar, uint32_t parity) {
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
    n_ptiles = p.n_ptiles_k;
    nb = p.gk.nb;
    words = p.gk.mask_words;
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

// One 128 x 128 tile: one box of 128 bytes per row (fp8) or two boxes of 64
// 16-bit columns.
template <class C>
__device__ __forceinline__ void load_tile(uint8_t* dst, const CUtensorMap* map, uint64_t* bar, int row,
                                          uint64_t policy) {
  mbar_arrive_expect_tx(bar, C::kTileBytes);
#pragma unroll
  for (int b = 0; b < C::kBoxes; ++b) tma_load_2d(dst + b * kBoxBytes, map, bar, b * 64, row, policy);
}

// Producer of one slot: takes units from the global counter, loads Q and then
// the K and V tiles of the KV list into rings of kKStages / kVStages buffers
// (K of tile t once S of tile t - stages is done, V once P V of tile
// t - stages is).  The fp8 path also passes each tile's block scales on.
template <class C>
__device__ void producer_loop(Smem<C>& sm, Slot<C>& sl, const AttnParams& p, const CUtensorMap* tq,
                              const CUtensorMap* tk, const CUtensorMap* tv) {
  const uint64_t pol_q = l2_policy_evict_first();
  const uint64_t pol_kv = l2_policy_evict_last();
  uint32_t c = 0, nk = 0, nv = 0;   // units, K tiles and V tiles issued
  const int S_int_k = p.gk.S_int;
  const int BN = p.B * p.N;
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
        itm.ntiles = p.gk.n_tiles;
      } else {
        mrow = p.mask + ((size_t)itm.bn * p.g.nb + (itm.qt - p.n_ptiles)) * p.gk.mask_words;
        int cnt = 0;
        for (int wd = 0; wd < p.gk.mask_words; ++wd) cnt += __popc(mrow[wd]);
        itm.ntiles = p.n_ptiles_k + cnt;
      }
    }
    sl.items[it] = itm;
    mbar_arrive(&sl.item_full[it]);
    if (itm.bn < 0) break;

    const int base = itm.bn * S_int_k;   // the unit's KV rows
    const float* sc_k = C::kFp8 ? p.scales + (size_t)BN * p.g.n_tiles + (size_t)itm.bn * p.gk.n_tiles : nullptr;
    const float* sc_v = C::kFp8 ? sc_k + (size_t)BN * p.gk.n_tiles : nullptr;
    if (c >= 1 && !wait1(sm, p, &sl.q_empty, ph(c - 1))) {
      ok = false;
      break;
    }
    if (!(p.skip_first_q && c == 0)) {
      if (C::kFp8) sl.q_scale = p.scales[(size_t)itm.bn * p.g.n_tiles + itm.qt];
      load_tile<C>(sl.q, tq, &sl.q_full, itm.bn * p.g.S_int + itm.qt * RF_BLOCK, pol_q);
    }
    ++c;
    KvIter kit;
    kit.init(base, p, mrow);
    for (int row = kit.next(); row >= 0 && ok; row = kit.next()) {
      const uint32_t ks = nk % C::kKStages, ku = nk / C::kKStages;
      if (ku >= 1 && !wait1(sm, p, &sl.k_empty[ks], ph(ku - 1))) {
        ok = false;
        break;
      }
      if (C::kFp8) {
        const int tile = (row - base) / RF_BLOCK;
        sl.kv_scale[ks][0] = sc_k[tile];
        sl.kv_scale[ks][1] = sc_v[tile];
      }
      load_tile<C>(sl.k[ks], tk, &sl.k_full[ks], row, pol_kv);
      ++nk;
      const uint32_t vs = nv % C::kVStages, vu = nv / C::kVStages;
      if (vu >= 1 && !wait1(sm, p, &sl.v_empty[vs], ph(vu - 1))) {
        ok = false;
        break;
      }
      load_tile<C>(sl.v[vs], tv, &sl.v_full[vs], row, pol_kv);
      ++nv;
    }
  }
  if (!ok) {
    // Let the copies already issued land before the CTA may exit (bounded by
    // time, not cut short by the abort flag).
    const uint64_t lim = p.wait_limit_ns / 4;
    if (c) rf_wait_time(&sl.q_full, ph(c - 1), lim);
    for (uint32_t st = 0; st < (uint32_t)C::kKStages; ++st) {
      const uint32_t n = (nk > st) ? (nk - st + C::kKStages - 1) / C::kKStages : 0;   // loads into stage st
      if (n) rf_wait_time(&sl.k_full[st], ph(n - 1), lim);
    }
    for (uint32_t st = 0; st < (uint32_t)C::kVStages; ++st) {
      const uint32_t n = (nv > st) ? (nv - st + C::kVStages - 1) / C::kVStages : 0;
      if (n) rf_wait_time(&sl.v_full[st], ph(n - 1), lim);
    }
  }
}

// ---------------------------------------------------------------- MMA issue
// Descriptor low words of the 128-byte swizzled operands; every descriptor
// used here shares one high word (stride 1024 B, sm_100 version, swizzle).
// A K step (16 16-bit or 32 8-bit elements) advances a K-major operand by
// 32 B (2 in the descriptor's 16-byte units); the second box of a 16-bit
// tile (columns 64..127) starts 16 KB further.  The issuing warp runs this
// code together; one elected lane issues.
template <class C>
__device__ __forceinline__ void issue_qk(uint32_t s_tmem, uint32_t q_lo, uint32_t k_lo, uint32_t hi) {
#pragma unroll
  for (int kk = 0; kk < C::kSteps; ++kk) {
    const uint32_t off = ((kk >> 2) * kBoxBytes + (kk & 3) * 32) >> 4;
    if (C::kFp8)
      mma_ss_lo_elect_f8(s_tmem, q_lo + off, k_lo + off, hi, C::kIdescQK, kk > 0);
    else
      mma_ss_lo_elect(s_tmem, q_lo + off, k_lo + off, hi, C::kIdescQK, kk > 0);
  }
}
// P V: a K step takes the next 8 TMEM columns of P (16 16-bit or 32 8-bit
// keys).  16-bit V is MN-major: 16 keys are 16 rows of 128 B further.  fp8 V
// is stored transposed (K-major): 32 keys are 32 B further.
template <class C>
__device__ __forceinline__ void issue_pv(uint32_t o_tmem, uint32_t p_tmem, uint32_t v_lo, uint32_t hi,
                                         bool accumulate) {
#pragma unroll
  for (int kk = 0; kk < C::kSteps; ++kk) {
    const uint32_t acc = (accumulate || kk > 0) ? 1u : 0u;
    if (C::kFp8)
      mma_ts_lo_elect_f8(o_tmem, p_tmem + kk * 8, v_lo + kk * 2, hi, C::kIdescPV, acc);
    else
      mma_ts_lo_elect(o_tmem, p_tmem + kk * 8, v_lo + kk * (2048 >> 4), hi, C::kIdescPV, acc);
  }
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
// P = 2^(s c + off) for the row's 128 scores s (already in registers), with
// the tile's sum of P; writes the packed P words.
template <class C>
__device__ __forceinline__ float exp_tile(const uint32_t (&s)[4][32], float c, float off, int p_valid,
                                          uint32_t (&pk)[C::kPCols]) {
  const uint64_t c2 = f2_pack(c, c);
  const uint64_t negm = f2_pack(off, off);
  const bool partial = p_valid < RF_BLOCK;
  uint64_t sum2[4] = {0, 0, 0, 0};
  float hold0 = 0.f, hold1 = 0.f;   // fp8: the first pair of a 4-key word
#pragma unroll
  for (int q4 = 0; q4 < 4; ++q4)
#pragma unroll
    for (int e = 0; e < 32; e += 2) {
      const int i = 16 * q4 + (e >> 1);     // pair index 0..63
      const uint64_t x2 = f2_fma(f2_pack(__uint_as_float(s[q4][e]), __uint_as_float(s[q4][e + 1])), c2, negm);
      uint64_t p2;
      if ((i % C::kPolyEvery) == C::kPolyEvery - 1) {
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
      if (C::kFp8) {
        if (i & 1)
          pk[i >> 1] = pack_e4m3x4(hold0, hold1, a0, a1);
        else {
          hold0 = a0;
          hold1 = a1;
        }
      } else {
        pk[i] = pack_half2<C::kF16>(a0, a1);
      }
    }
  float s0, s1, s2, s3;
  f2_unpack(f2_add(sum2[0], sum2[1]), s0, s1);
  f2_unpack(f2_add(sum2[2], sum2[3]), s2, s3);
  return (s0 + s1) + (s2 + s3);
}

template <class C>
__device__ __forceinline__ void load_scores(uint32_t tS, int p_valid, uint32_t (&s)[4][32]) {
#pragma unroll
  for (int q4 = 0; q4 < 4; ++q4) tmem_ld32(tS + 32 * q4, s[q4]);
  tmem_wait_ld();
#pragma unroll
  for (int q4 = 0; q4 < 4; ++q4) reg_fence32(s[q4]);
  if (p_valid < RF_BLOCK) {
#pragma unroll
    for (int q4 = 0; q4 < 4; ++q4)
#pragma unroll
      for (int e = 0; e < 32; ++e)
        if (32 * q4 + e >= p_valid) s[q4][e] = __float_as_uint(-CUDART_INF_F);
  }
}

__device__ __forceinline__ float row_max(const uint32_t (&s)[4][32]) {
  float mx8[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) mx8[i] = -CUDART_INF_F;
#pragma unroll
  for (int q4 = 0; q4 < 4; ++q4)
#pragma unroll
    for (int e = 0; e < 32; e += 2)
      mx8[(e >> 1) & 7] = max3f(mx8[(e >> 1) & 7], __uint_as_float(s[q4][e]), __uint_as_float(s[q4][e + 1]));
  return max3f(max3f(mx8[0], mx8[1], mx8[2]), max3f(mx8[3], mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7]));
}

// Thread = query row.  Reads the row's 128 scores from S and writes P =
// 2^(s c - m_use + lr) over the first columns of S (64 words of two 16-bit
// values, or (fp8) 32 words of four e4m3 codes), adding the tile's sum of P
// times ir to l.  The running max m_use (log2 units) is set by the unit's
// first tile; later tiles use it as it stands and look at their own maximum
// only when their sum shows a P above the format's limit (sum > kSumLimit,
// or not finite): then the scores are read again, m_use moves up to the
// tile's maximum if that exceeds it by more than the threshold (rescaling O
// and l), and P is computed again.  `p_valid` < 128 masks the keys past the
// prefix's end.
template <class C>
__device__ __forceinline__ void softmax_tile(uint32_t tS, uint32_t tO, bool first, int p_valid, float c, float lr,
                                             float ir, float& m_use, float& l) {
  // P above this sum may exceed 448 (e4m3) / lose fp32 headroom (16-bit)
  constexpr float kSumLimit = C::kFp8 ? 448.f : 65536.f;
  uint32_t s[4][32];
  uint32_t pk[C::kPCols];
  load_scores<C>(tS, p_valid, s);
  float alpha = 1.f;
  bool rescale = false;
  float tsum;
  if (first) {
    m_use = row_max(s) * c;
    tsum = exp_tile<C>(s, c, lr - m_use, p_valid, pk);
  } else {
    tsum = exp_tile<C>(s, c, lr - m_use, p_valid, pk);
    if (__any_sync(0xFFFFFFFFu, !(tsum <= kSumLimit))) {
      load_scores<C>(tS, p_valid, s);
      const float mx_s = row_max(s) * c;
      if (mx_s > m_use + kRescaleThreshold) {
        alpha = ex2_approx(m_use - mx_s);
        m_use = mx_s;
        rescale = true;
      }
      tsum = exp_tile<C>(s, c, lr - m_use, p_valid, pk);
    }
  }
  l = l * alpha + tsum * ir;
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
#pragma unroll
  for (int w = 0; w < C::kPCols; w += 32) tmem_st32(tS + w, *reinterpret_cast<uint32_t(*)[32]>(&pk[w]));
  tmem_wait_st();
  tc_fence_before();
}

// ---------------------------------------------------------------- one slot
// The slot's four warps compute the softmax of each tile (thread = query row
// = TMEM lane) and write the unit's output; the first of them also issues
// the slot's MMAs: S = Q K^T of a tile once the P V of the previous tile is
// done (P lives in the S columns), and P V of a tile once all four warps
// have written P (the rendezvous after each tile).
template <class C>
__device__ void slot_loop(Smem<C>& sm, Slot<C>& sl, const AttnParams& p, uint32_t tmem_slot, int bar_id) {
  const int quad = (threadIdx.x >> 5) & 3;
  const bool issuer = (quad == 0);
  const int row = quad * 32 + (threadIdx.x & 31);   // query row == TMEM lane
  const uint32_t lane_base = tmem_slot + ((uint32_t)(quad * 32) << 16);
  const uint32_t tS = lane_base, tO = lane_base + 128;
  const uint32_t s_tmem = tmem_slot, o_tmem = tmem_slot + 128;
  const uint32_t hi = (uint32_t)(make_sdesc_sw128(0, 16, 1024) >> 32);
  const uint32_t q_lo = (uint32_t)make_sdesc_sw128(smem_u32(sl.q), 16, 1024);
  const uint32_t k_lo0 = (uint32_t)make_sdesc_sw128(smem_u32(sl.k[0]), 16, 1024);
  const uint32_t v_lo0 = (uint32_t)make_sdesc_sw128(smem_u32(sl.v[0]), C::kFp8 ? 16 : kBoxBytes, 1024);
  uint32_t c = 0, t = 0;   // units and tiles of this slot
  bool ok = true;
  bool issued = false;     // the issuer has MMAs that may still run
  float q_scale = 1.f;     // fp8: the unit's Q block scale (issuer)
  float unit_vmax = 1.f;   // fp8: the largest V block scale of the unit's head (issuer)

  // S = Q K^T of tile tt (issuer warp): K tile tt must have landed and the
  // P V of tile tt - 1 must be done.  Then the tile's fp8 factors go to
  // ts[tt & 1], and the issuer's arrival on s_full publishes them.
  auto qk = [&](uint32_t tt, bool last_of_unit) -> bool {
    const uint32_t ks = tt % C::kKStages;
    if (!waitw(sm, p, &sl.k_full[ks], ph(tt / C::kKStages))) return false;
    // read before the MMAs: once they finish, the producer may refill the stage
    const float sk = C::kFp8 ? sl.kv_scale[ks][0] : 0.f, sv = C::kFp8 ? sl.kv_scale[ks][1] : 0.f;
    if (tt >= 1 && !waitw(sm, p, &sl.pv_done, ph(tt - 1))) return false;
    tc_fence_after();
    issue_qk<C>(s_tmem, q_lo, k_lo0 + ks * (C::kTileBytes >> 4), hi);
    mma_commit_elect(&sl.s_full);
    mma_commit_elect(&sl.k_empty[ks]);
    if (last_of_unit) mma_commit_elect(&sl.q_empty);
    issued = true;
    if ((threadIdx.x & 31) == 0) {
      if (C::kFp8) {
        const float vmax = unit_vmax;
        TileScale f;
        f.c = p.scale_log2 * q_scale * sk;
        const bool use_r = sv > 0.f && vmax > 0.f;   // an all-zero V block adds nothing whatever P is
        f.lr = use_r ? __log2f(sv / vmax) : 0.f;
        f.ir = use_r ? vmax / sv : 1.f;
        f.pad = 0.f;
        sl.ts[tt & 1] = f;
      }
      mbar_arrive(&sl.s_full);
    }
    __syncwarp();
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
    if (issuer) {
      ok = waitw(sm, p, &sl.q_full, ph(c));
      if (C::kFp8 && ok) {
        q_scale = sl.q_scale;
        unit_vmax = p.vmax[itm.bn];
      }
      if (ok) ok = qk(t, itm.ntiles == 1);
    }
    const float out_scale = C::kFp8 ? p.vmax[itm.bn] : 1.f;

    float m_use = -CUDART_INF_F, l = 0.f;
    for (int j = 0; j < itm.ntiles; ++j, ++t) {
      if (ok) ok = waitw(sm, p, &sl.s_full, ph(t));
      if (ok) {
        tc_fence_after();
        const int p_valid = (p.p_rem_k != 0 && j == p.n_ptiles_k - 1) ? p.p_rem_k : RF_BLOCK;
        if (C::kFp8) {
          const TileScale f = sl.ts[t & 1];
          softmax_tile<C>(tS, tO, j == 0, p_valid, f.c, f.lr, f.ir, m_use, l);
        } else {
          softmax_tile<C>(tS, tO, j == 0, p_valid, p.scale_log2, 0.f, 1.f, m_use, l);
        }
      }
      ok = slot_vote(bar_id, ok);
      if (!ok) break;
      if (issuer) {
        const uint32_t vs = t % C::kVStages;
        ok = waitw(sm, p, &sl.v_full[vs], ph(t / C::kVStages));
        if (ok) {
          tc_fence_after();
          issue_pv<C>(o_tmem, s_tmem, v_lo0 + vs * (C::kTileBytes >> 4), hi, j > 0);
          mma_commit_elect(&sl.pv_done);
          mma_commit_elect(&sl.v_empty[vs]);
          if (j + 1 < itm.ntiles) ok = qk(t + 1, j + 2 == itm.ntiles);
        }
      }
    }
    // epilogue: O * out_scale / l of this unit once its last P V is done
    if (ok) ok = waitw(sm, p, &sl.pv_done, ph(t - 1));
    if (ok) {
      tc_fence_after();
      const float rl = out_scale / l;
      const int b = itm.bn / p.N, nh = itm.bn - b * p.N;
      const int src = rf_src_of_row(p.g, itm.qt * RF_BLOCK + row);
      uint16_t* dst = src >= 0
                          ? static_cast<uint16_t*>(p.out) + rf_token_offset(p.layout, p.B, p.S, p.N, b, nh, src)
                          : nullptr;
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
            w[e] = pack_half2<C::kF16>(__uint_as_float(o[2 * e]) * rl, __uint_as_float(o[2 * e + 1]) * rl);
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

template <class C>
__global__ void __launch_bounds__(kThreads, 1)
    attn_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const AttnParams p) {
  extern __shared__ uint8_t smem_raw[];
  Smem<C>& sm = *reinterpret_cast<Smem<C>*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int z = 0; z < kSlots; ++z) {
      Slot<C>& sl = sm.slot[z];
      mbar_init(&sl.q_full, 1);
      mbar_init(&sl.q_empty, 1);
      for (int i = 0; i < C::kKStages; ++i) {
        mbar_init(&sl.k_full[i], 1);
        mbar_init(&sl.k_empty[i], 1);
      }
      for (int i = 0; i < C::kVStages; ++i) {
        mbar_init(&sl.v_full[i], 1);
        mbar_init(&sl.v_empty[i], 1);
      }
      mbar_init(&sl.s_full, 2);   // the MMA commit and the issuer's arrival
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
    slot_loop<C>(sm, sm.slot[z], p, tmem + 256 * z, 1 + z);
  } else {
    regs_decrease<kRegsControl>();
    if (warp == 8 && lane == 0) producer_loop<C>(sm, sm.slot[0], p, &tm_q, &tm_k, &tm_v);
    if (warp == 9 && lane == 0) producer_loop<C>(sm, sm.slot[1], p, &tm_q, &tm_k, &tm_v);
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

// [rows, 128] elements of `elem_bytes` (2: bf16/fp16, 1: e4m3 codes),
// row-major; boxes of 128 rows x 128 bytes, 128-byte swizzle.
bool make_tile_map(CUtensorMap* map, const void* base, uint64_t rows, CUtensorMapDataType type, int elem_bytes) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[2] = {RF_HEAD_DIM, rows};
  const cuuint64_t strides[1] = {(cuuint64_t)RF_HEAD_DIM * elem_bytes};
  const cuuint32_t box[2] = {(cuuint32_t)(128 / elem_bytes), RF_BLOCK};
  const cuuint32_t estr[2] = {1, 1};
  return enc(map, type, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

AttnParams make_params(const uint32_t* mask, int layout, int B, int S, int N, const rf_plan_t& g,
                       const rf_plan_t& gk, float scale, void* out, int* counter, int* status, const AttnDebug& dbg) {
  AttnParams p;
  p.g = g;
  p.gk = gk;
  p.B = B;
  p.S = S;
  p.N = N;
  p.layout = layout;
  p.total_items = B * N * g.n_tiles;
  p.n_ptiles = g.P_pad / RF_BLOCK;
  p.n_ptiles_k = gk.P_pad / RF_BLOCK;
  p.p_rem_k = gk.P % RF_BLOCK;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.mask = mask;
  p.scales = nullptr;
  p.vmax = nullptr;
  p.counter = counter;
  p.status = status;
  p.out = out;
  p.wait_limit_ns = dbg.wait_limit_ns > 0 ? (uint64_t)dbg.wait_limit_ns : kWaitLimitNs;
  p.skip_first_q = dbg.skip_first_q;
  return p;
}

template <class C>
cudaError_t launch_cfg(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const AttnParams& p,
                       cudaStream_t stream) {
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  const size_t smem = sizeof(Smem<C>) + 1024;
  e = cudaFuncSetAttribute(attn_kernel<C>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  e = cudaMemsetAsync(p.counter, 0, sizeof(int), stream);
  if (e != cudaSuccess) return e;
  const int grid = std::min(sms, p.total_items);
  attn_kernel<C><<<grid, kThreads, smem, stream>>>(tq, tk, tv, p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attention(const void* q_int, const void* k_int, const void* v_int, const uint32_t* mask,
                             int dtype, int layout, int B, int S, int N, const rf_plan_t& g, const rf_plan_t& gk,
                             float scale, void* out, int* counter, int* status, const AttnDebug& dbg,
                             cudaStream_t stream) {
  const uint64_t rows_q = (uint64_t)B * N * g.S_int, rows_k = (uint64_t)B * N * gk.S_int;
  const bool f16 = dtype == RF_F16;
  const CUtensorMapDataType type = f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  CUtensorMap tq, tk, tv;
  if (!make_tile_map(&tq, q_int, rows_q, type, 2) || !make_tile_map(&tk, k_int, rows_k, type, 2) ||
      !make_tile_map(&tv, v_int, rows_k, type, 2))
    return cudaErrorInvalidValue;
  const AttnParams p = make_params(mask, layout, B, S, N, g, gk, scale, out, counter, status, dbg);
  return f16 ? launch_cfg<Cfg<true, false>>(tq, tk, tv, p, stream)
             : launch_cfg<Cfg<false, false>>(tq, tk, tv, p, stream);
}

cudaError_t launch_attention_fp8(const uint8_t* q8, const uint8_t* k8, const uint8_t* v8, const float* scales,
                                 const float* vmax, const uint32_t* mask, int dtype, int layout, int B, int S, int N,
                                 const rf_plan_t& g, const rf_plan_t& gk, float scale, void* out, int* counter,
                                 int* status, const AttnDebug& dbg, cudaStream_t stream) {
  const uint64_t rows_q = (uint64_t)B * N * g.S_int, rows_k = (uint64_t)B * N * gk.S_int;
  CUtensorMap tq, tk, tv;
  if (!make_tile_map(&tq, q8, rows_q, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1) ||
      !make_tile_map(&tk, k8, rows_k, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1) ||
      !make_tile_map(&tv, v8, rows_k, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1))
    return cudaErrorInvalidValue;
  AttnParams p = make_params(mask, layout, B, S, N, g, gk, scale, out, counter, status, dbg);
  p.scales = scales;
  p.vmax = vmax;
  return dtype == RF_F16 ? launch_cfg<Cfg<true, true>>(tq, tk, tv, p, stream)
                         : launch_cfg<Cfg<false, true>>(tq, tk, tv, p, stream);
}

}  // namespace rf
