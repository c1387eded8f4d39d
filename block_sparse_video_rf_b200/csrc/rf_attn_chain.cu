// Block-sparse flash attention on sm_100a tensor cores (K3), 16-bit path:
// one query tile per CTA, three key tiles in flight.
//
// Work unit and KV list as in rf_attn_common.cuh (lite_boost.ops.
// sparse_attention, rf_v2 pipeline; vllm-omni "RainFusion Attention",
// intro).  A CTA (one per SM, persistent) runs one unit at a time, but its
// key tiles run in three chains: tile j of a unit has its scores S in
// tensor-memory buffer j % 3, and three warp sets share the softmaxes (fp8:
// set j % 3 takes tile j; 16-bit: two sets take a tile's two halves of 64
// keys at once), so softmaxes and the MMAs of the other tiles overlap.  All three add
// into one O, so they share one running maximum: the row maximum of the
// unit's first tile (log2 units), published through shared memory.  P is
// 2^(s c - m) with that m throughout the unit (no per-tile maximum, no
// rescale); a tile whose sum of P passes the headroom of the P type (2^64
// for bf16, 65504 for fp16) marks its rows, and the whole unit is handed to
// the second pass (attn_kernel in list mode, which rescales as it goes)
// instead of being written.  Each set keeps the sum l of its own tasks; the
// set of the unit's last task adds the three sums in a fixed order and
// writes O / l to the caller's layout.  Which set takes which task depends
// on the task's place in its unit only, so results do not depend on which
// CTA ran the unit.
//
// Warps (512 threads):
//   0-11  softmax sets 0, 1, 2 (four warps each, thread = query row = TMEM
//         lane); the set of a unit's last task also writes the unit's output.
//   12    TMA producer of Q and K (one thread): takes units from the global
//         counter and publishes them to the other roles through a queue.
//   13    TMA producer of V (one thread).
//   14    P V issuer (one elected lane): O += P V of each tile once P is
//         written.
//   15    S issuer: S = Q K^T of each tile once the P V of the buffer's
//         previous tile is done (P lives in the S columns); owns the tensor
//         memory.
// Shared memory: Q (32 KB), rings of three K and three V tiles (96 KB each),
// 128-byte swizzled boxes of 128 rows x 128 bytes; K of the CTA's tile g
// loads once the S of tile g - 3 is done, V once the P V of tile g - 3 is.
// Tensor memory (512 columns): S_c at [128 c, 128 c + 128) for c = 0, 1, 2,
// O at [384, 512).  P of a tile's keys 64 h .. 64 h + 63 overwrites S
// columns already read: 16-bit, the first 32 of those keys' own columns
// (from 128 c + 64 h); e4m3, 16 columns from 128 c + 16 h.
#include <cstring>

#include "rf_attn_common.cuh"

namespace rf {

namespace {

constexpr int kCThreads = 512;
constexpr int kSets = 3;                      // S buffers = softmax warp sets
// Q buffers and K / V tiles in flight.  16-bit (32 KB tiles): shared memory
// holds 7 tiles, one Q, three K and three V (a second Q buffer, taken from
// the V ring, measured slower: the bubble at a unit change costs less than a
// shallower V ring).  fp8 (16 KB tiles): two Q, four K and four V.
template <class C>
struct ChainShape {
  static constexpr int kQBufs = C::kFp8 ? 2 : 1;
  static constexpr int kKRing = C::kFp8 ? 4 : 3;
  static constexpr int kVRing = C::kFp8 ? 4 : 3;
};
constexpr int kItemQ = 8;                     // depth of the unit queue
// Softmax tasks per key tile after a unit's first: 16-bit tiles are split
// into two halves of 64 keys done by two sets at once, fp8 tiles are not.
template <class C>
constexpr int kTaskSplit = C::kFp8 ? 1 : 2;
// Column of P of a tile's keys 64..127 within its buffer.  Split tiles keep
// each half's P inside the half's own S columns, so the two sets never touch
// each other's scores; whole tiles pack P into the first columns.
template <class C>
constexpr uint32_t kPHalfCol = kTaskSplit<C> == 2 ? 64u : (C::kFp8 ? 16u : 32u);
constexpr uint32_t kCTmemCols = 512;
constexpr int kWarpKProd = 12, kWarpVProd = 13, kWarpPV = 14, kWarpQK = 15;
constexpr int kItemReaders = 3 + 4 * kSets;   // V producer, the two MMA warps, softmax warps
constexpr int kMaxSmem = 232448;              // 227 KB: the most dynamic shared memory a CTA may have

template <class C, class CS = ChainShape<C>>
struct __align__(1024) ChainSmem {
  uint8_t q[CS::kQBufs][C::kTileBytes];
  uint8_t k[CS::kKRing][C::kTileBytes];
  uint8_t v[CS::kVRing][C::kTileBytes];
  uint64_t q_full[CS::kQBufs], q_empty[CS::kQBufs];
  uint64_t k_full[CS::kKRing], k_empty[CS::kKRing], v_full[CS::kVRing], v_empty[CS::kVRing];
  uint64_t s_full[kSets];     // S of the set's next tile is in TMEM (MMA commit; fp8: and the S warp's
                              // arrival once the tile's factors are in ts)
  uint64_t p_full[kSets];     // P of the buffer's tile written (one arrival per warp and task)
  uint64_t pv_done[kSets];    // P V of the set's tile done (MMA commit)
  uint64_t o_full;            // the last P V of a unit done (MMA commit)
  uint64_t o_free;            // the unit's output has been read out of O (4 warps)
  uint64_t m_full, m_empty;   // the unit's maximum published (4 warps) / taken by every warp (12)
  uint64_t l_full, l_empty;   // every set's row sums posted (12) / read by the output set (4)
  uint64_t item_full[kItemQ], item_empty[kItemQ];
  uint64_t drain[2];          // the two MMA warps' last commits when they leave early
  Item items[kItemQ];
  float m_sh[RF_BLOCK];
  float l_sh[kSets][RF_BLOCK];
  float kv_scale[CS::kKRing][2];   // fp8: {sk, sv} of the tile in each K slot (K producer, with k_full)
  TileScale ts[kSets];             // fp8: factors of each buffer's tile (S warp, with s_full)
  uint32_t tmem_base;
  int abort;
};
static_assert(sizeof(ChainSmem<Cfg<false, false>>) <= kMaxSmem, "shared memory of the chain kernel");
static_assert(sizeof(ChainSmem<Cfg<false, true>>) <= kMaxSmem, "shared memory of the chain kernel");

// Sum of P above which a tile's unit goes to the second pass: P must stay
// finite in its type (bf16 to 2^127: the limit 2^64 keeps O and l far from
// fp32 overflow; fp16 to 65504; e4m3 to 448 before it saturates), and every
// P is at most the sum.
template <class C>
__device__ __forceinline__ float sum_limit(const AttnParams& p) {
  return p.sum_limit > 0.f ? p.sum_limit : (C::kFp8 ? 448.f : C::kF16 ? 65504.f : 18446744073709551616.f);
}

__device__ __forceinline__ const uint32_t* mask_row(const AttnParams& p, const Item& itm) {
  return is_dense_tile(p, itm.qt) ? nullptr
                                  : p.mask + ((size_t)itm.bn * p.g.nb + (itm.qt - p.n_ptiles)) * p.gk.mask_words;
}

// Rendezvous of one set's four warps (named barrier 1 + set) returning the
// AND (or the OR) of a predicate over its 128 threads.
__device__ __forceinline__ bool set_and(int set, bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred a, b;\n\tsetp.ne.u32 a, %1, 0;\n\t"
      "bar.red.and.pred b, %2, 128, a;\n\tselp.u32 %0, 1, 0, b;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)v), "r"(1 + set)
      : "memory");
  return r != 0;
}
__device__ __forceinline__ bool set_or(int set, bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred a, b;\n\tsetp.ne.u32 a, %1, 0;\n\t"
      "bar.red.or.pred b, %2, 128, a;\n\tselp.u32 %0, 1, 0, b;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)v), "r"(1 + set)
      : "memory");
  return r != 0;
}

// ---------------------------------------------------------------- producers
// Q and K: takes units from the global counter, publishes each to the unit
// queue, loads its Q tile (once every S of the previous unit is done) and
// its K tiles into the ring.
template <class C>
__device__ void kprod_loop(ChainSmem<C>& sm, const AttnParams& p, const CUtensorMap* tq, const CUtensorMap* tk) {
  using CS = ChainShape<C>;
  const int BN = p.B * p.N;
  const uint64_t pol_q = l2_policy_evict_first();
  const uint64_t pol_kv = l2_policy_evict_last();
  uint32_t u = 0, nk = 0;   // units published, K tiles issued
  uint32_t nq[CS::kQBufs] = {};   // Q loads issued into each buffer
  bool ok = true;
  while (ok) {
    const int w = atomicAdd(p.counter, 1);
    const uint32_t qi = u % kItemQ;
    if (u >= kItemQ && !wait1(&sm.abort, p, &sm.item_empty[qi], ph(u / kItemQ - 1))) {
      ok = false;
      break;
    }
    const uint32_t* mrow;
    Item itm = make_item(p, unit_of(p, w), mrow);
    const int own = own_tile(p, itm, mrow);
    itm.partial = partial_place(p, own);
    sm.items[qi] = itm;
    mbar_arrive(&sm.item_full[qi]);
    if (itm.bn < 0) break;
    const uint32_t qb = u % CS::kQBufs;
    if (u >= (uint32_t)CS::kQBufs && !wait1(&sm.abort, p, &sm.q_empty[qb], ph(u / CS::kQBufs - 1))) {
      ok = false;
      break;
    }
    if (!(p.skip_first_q && u == 0)) {
      load_tile<C>(sm.q[qb], tq, &sm.q_full[qb], itm.bn * p.g.S_int + itm.qt * RF_BLOCK, pol_q);
      ++nq[qb];
    }
    ++u;
    const int base = itm.bn * p.gk.S_int;   // the unit's KV rows
    const float* sc_k = C::kFp8 ? p.scales + (size_t)BN * p.g.n_tiles + (size_t)itm.bn * p.gk.n_tiles : nullptr;
    const float* sc_v = C::kFp8 ? sc_k + (size_t)BN * p.gk.n_tiles : nullptr;
    KvIter kit;
    kit.init(base, p, mrow, own);
    for (int row = kit.next(); row >= 0; row = kit.next()) {
      const uint32_t s = nk % CS::kKRing, n = nk / CS::kKRing;
      if (n >= 1 && !wait1(&sm.abort, p, &sm.k_empty[s], ph(n - 1))) {
        ok = false;
        break;
      }
      if (C::kFp8) {   // published by the arrival in load_tile, read under k_full
        const int tile = (row - base) / RF_BLOCK;
        sm.kv_scale[s][0] = sc_k[tile];
        sm.kv_scale[s][1] = sc_v[tile];
      }
      load_tile<C>(sm.k[s], tk, &sm.k_full[s], row, pol_kv);
      ++nk;
    }
  }
  if (!ok) {
    // Let the copies already issued land before the CTA may exit (bounded by
    // time, not cut short by the abort flag).
    const uint64_t lim = p.wait_limit_ns / 4;
    for (uint32_t b = 0; b < (uint32_t)CS::kQBufs; ++b)
      if (nq[b]) rf_wait_time(&sm.q_full[b], ph(nq[b] - 1), lim);
    for (uint32_t st = 0; st < (uint32_t)CS::kKRing; ++st) {
      const uint32_t n = (nk > st) ? (nk - st + CS::kKRing - 1) / CS::kKRing : 0;
      if (n) rf_wait_time(&sm.k_full[st], ph(n - 1), lim);
    }
  }
}

// V: follows the unit queue and loads the V tiles into their ring.
template <class C>
__device__ void vprod_loop(ChainSmem<C>& sm, const AttnParams& p, const CUtensorMap* tv) {
  using CS = ChainShape<C>;
  const uint64_t pol_kv = l2_policy_evict_last();
  uint32_t nv = 0;
  bool ok = true;
  for (uint32_t u = 0; ok; ++u) {
    const uint32_t qi = u % kItemQ;
    if (!wait1(&sm.abort, p, &sm.item_full[qi], ph(u / kItemQ))) {
      ok = false;
      break;
    }
    const Item itm = sm.items[qi];
    mbar_arrive(&sm.item_empty[qi]);
    if (itm.bn < 0) break;
    KvIter kit;
    const uint32_t* mrow = mask_row(p, itm);
    kit.init(itm.bn * p.gk.S_int, p, mrow, own_tile(p, itm, mrow));
    for (int row = kit.next(); row >= 0; row = kit.next()) {
      const uint32_t s = nv % CS::kVRing, n = nv / CS::kVRing;
      if (n >= 1 && !wait1(&sm.abort, p, &sm.v_empty[s], ph(n - 1))) {
        ok = false;
        break;
      }
      load_tile<C>(sm.v[s], tv, &sm.v_full[s], row, pol_kv);
      ++nv;
    }
  }
  if (!ok) {
    const uint64_t lim = p.wait_limit_ns / 4;
    for (uint32_t st = 0; st < (uint32_t)CS::kVRing; ++st) {
      const uint32_t n = (nv > st) ? (nv - st + CS::kVRing - 1) / CS::kVRing : 0;
      if (n) rf_wait_time(&sm.v_full[st], ph(n - 1), lim);
    }
  }
}

// ---------------------------------------------------------------- MMA issuers
// Tile j of a unit has its S in buffer j % 3.  Two warps issue into the one
// tensor pipe, so that neither product waits behind the other's hand-offs:
// the S warp issues S = Q K^T of each tile once the P V of the buffer's
// previous tile is done (P lives in the S columns), the P V warp issues
// O += P V of each tile once its P is written.  Each warp commits its own
// MMAs.  On an abort each waits (bounded) for its MMAs before leaving.
template <class C>
__device__ void qk_loop(ChainSmem<C>& sm, const AttnParams& p, uint32_t tmem) {
  using CS = ChainShape<C>;
  const uint32_t hi = (uint32_t)(make_sdesc_sw128(0, 16, 1024) >> 32);
  const uint32_t q_lo0 = (uint32_t)make_sdesc_sw128(smem_u32(sm.q[0]), 16, 1024);
  const uint32_t k_lo0 = (uint32_t)make_sdesc_sw128(smem_u32(sm.k[0]), 16, 1024);
  uint32_t uses[kSets] = {0, 0, 0};   // S tiles issued into each buffer
  uint32_t gq = 0;                    // the CTA's tiles issued (K ring position)
  bool ok = true, issued = false;
  for (uint32_t u = 0; ok; ++u) {
    const uint32_t qi = u % kItemQ;
    if (!waitw(&sm.abort, p, &sm.item_full[qi], ph(u / kItemQ))) {
      ok = false;
      break;
    }
    const Item itm = sm.items[qi];
    arrive_w(&sm.item_empty[qi]);
    if (itm.bn < 0) break;
    const uint32_t qb = u % CS::kQBufs;
    const uint32_t q_lo = q_lo0 + qb * (C::kTileBytes >> 4);
    if (!waitw(&sm.abort, p, &sm.q_full[qb], ph(u / CS::kQBufs))) {
      ok = false;
      break;
    }
    // fp8: the unit's Q block scale and the head's largest V block scale
    const float sq = C::kFp8 ? p.scales[(size_t)itm.bn * p.g.n_tiles + itm.qt] : 0.f;
    const float vmax = C::kFp8 ? p.vmax[itm.bn] : 0.f;
    for (int j = 0; j < itm.ntiles; ++j, ++gq) {
      const int c = j % kSets;
      const uint32_t ks = gq % CS::kKRing;
      // K lands tiles ahead; the buffer's previous P V is the wait that counts
      if (!waitw(&sm.abort, p, &sm.k_full[ks], ph(gq / CS::kKRing))) {
        ok = false;
        break;
      }
      // read before the MMAs: once they finish, the producer may refill the slot
      const float sk = C::kFp8 ? sm.kv_scale[ks][0] : 0.f, sv = C::kFp8 ? sm.kv_scale[ks][1] : 0.f;
      if (uses[c] >= 1 && !waitw(&sm.abort, p, &sm.pv_done[c], ph(uses[c] - 1))) {
        ok = false;
        break;
      }
      tc_fence_after();
      issue_qk<C>(tmem + 128 * c, q_lo, k_lo0 + ks * (C::kTileBytes >> 4), hi);
      mma_commit_elect(&sm.s_full[c]);
      mma_commit_elect(&sm.k_empty[ks]);
      if (j == itm.ntiles - 1) mma_commit_elect(&sm.q_empty[qb]);
      issued = true;
      ++uses[c];
      if (C::kFp8) {
        // the set of buffer c read the previous tile's factors before its P,
        // which came before that tile's P V
        if ((threadIdx.x & 31) == 0) {
          sm.ts[c] = tile_scale(p, sq, sk, sv, vmax);
          mbar_arrive(&sm.s_full[c]);
        }
        __syncwarp();
      }
    }
  }
  if (!ok && issued) {
    mma_commit_elect(&sm.drain[0]);
    rf_wait_time(&sm.drain[0], 0, p.wait_limit_ns / 4);
    __syncwarp();
  }
}

template <class C>
__device__ void pv_loop(ChainSmem<C>& sm, const AttnParams& p, uint32_t tmem) {
  using CS = ChainShape<C>;
  const uint32_t hi = (uint32_t)(make_sdesc_sw128(0, 16, 1024) >> 32);
  const uint32_t v_lo0 = (uint32_t)make_sdesc_sw128(smem_u32(sm.v[0]), C::kFp8 ? 16 : kBoxBytes, 1024);
  const uint32_t o_tmem = tmem + 384;
  uint32_t uses[kSets] = {0, 0, 0};   // P V tiles issued from each buffer
  uint32_t gp = 0;                    // the CTA's tiles issued (V ring position)
  bool ok = true, issued = false;
  for (uint32_t u = 0; ok; ++u) {
    const uint32_t qi = u % kItemQ;
    if (!waitw(&sm.abort, p, &sm.item_full[qi], ph(u / kItemQ))) {
      ok = false;
      break;
    }
    const Item itm = sm.items[qi];
    arrive_w(&sm.item_empty[qi]);
    if (itm.bn < 0) break;
    for (int j = 0; j < itm.ntiles; ++j, ++gp) {
      const int c = j % kSets;
      const uint32_t vs = gp % CS::kVRing;
      if (!waitw(&sm.abort, p, &sm.v_full[vs], ph(gp / CS::kVRing))) {
        ok = false;
        break;
      }
      // the previous unit's output must have left O before its first P V
      if (j == 0 && u >= 1 && !waitw(&sm.abort, p, &sm.o_free, ph(u - 1))) {
        ok = false;
        break;
      }
      if (!waitw(&sm.abort, p, &sm.p_full[c], ph(uses[c]))) {
        ok = false;
        break;
      }
      tc_fence_after();
      issue_pv<C>(o_tmem, tmem + 128 * c, v_lo0 + vs * (C::kTileBytes >> 4), hi, j > 0, kPHalfCol<C>);
      mma_commit_elect(&sm.pv_done[c]);
      mma_commit_elect(&sm.v_empty[vs]);
      if (j == itm.ntiles - 1) mma_commit_elect(&sm.o_full);
      issued = true;
      ++uses[c];
    }
  }
  if (!ok && issued) {
    mma_commit_elect(&sm.drain[1]);
    rf_wait_time(&sm.drain[1], 0, p.wait_limit_ns / 4);
    __syncwarp();
  }
}

// ---------------------------------------------------------------- softmax sets
// Row maximum of a tile's 128 scores (-inf past p_valid).
__device__ __forceinline__ float tile_max(uint32_t tS, int p_valid) {
  float mx = -CUDART_INF_F;
#pragma unroll 1
  for (int h = 0; h < 2; ++h) {
    uint32_t s[2][32];
    load_scores<2>(tS + 64 * h, p_valid - 64 * h, s);
    mx = fmaxf(mx, row_max<2>(s));
  }
  return mx;
}

// P = 2^(s c + off) of half h (keys 64 h .. 64 h + 63) of a tile's row.  P
// goes to the 32 (16-bit, two per column) or 16 (e4m3, four per column)
// columns from kPHalfCol h of the tile's buffer, which are read already.
// Returns the half's sum of P; the caller waits for the store.
template <class C>
__device__ __forceinline__ float half_softmax(uint32_t tS, int h, int p_valid, float c, float off) {
  uint32_t s[2][32];
  load_scores<2>(tS + 64 * h, p_valid - 64 * h, s);
  float sum;
  if constexpr (C::kFp8) {
    uint32_t pk[16];
    sum = exp_scores<C, 2>(s, c, off, p_valid - 64 * h, pk);
    tmem_st16(tS + kPHalfCol<C> * h, pk);
  } else {
    uint32_t pk[32];
    sum = exp_scores<C, 2>(s, c, off, p_valid - 64 * h, pk);
    tmem_st32(tS + kPHalfCol<C> * h, pk);
  }
  return sum;
}
// Both halves of a tile's row, one after the other.  Returns the sum of P.
template <class C>
__device__ __forceinline__ float tile_softmax(uint32_t tS, int p_valid, float c, float off) {
  float tsum = 0.f;
#pragma unroll 1
  for (int h = 0; h < 2; ++h) tsum += half_softmax<C>(tS, h, p_valid, c, off);
  tmem_wait_st();
  return tsum;
}

// Set `set` (warps 4 set .. 4 set + 3).  Tile j of a unit has its scores in
// buffer j % 3.  Set 0 takes the unit's first tile whole: its row maximum
// becomes the unit's, published through shared memory, then its P.  16-bit:
// every later tile is two tasks, its halves of 64 keys, so that two sets work
// on one tile at once and a tile's P is ready sooner, which shortens the
// chain of S, softmax, P V and the next S into the tile's buffer; task
// t = 2 (j - 1) + h goes to set (t + 1) % 3.  fp8, whose softmax costs more
// issue slots per key, gains nothing from the shorter chain and loses the
// second rendezvous: every later tile is one task, t = j - 1, so tile j goes
// to set j % 3.  Each set takes its tasks in order.  A set keeps the sum l
// of its tasks' P; the set of the unit's last task adds the three sums in a
// fixed order and writes the output.  Which set takes which task depends on
// the task's place in its unit only, so results do not depend on which CTA
// ran a unit.
// The set's four warps meet at a named barrier once per task and carry any
// failed wait to it, so they leave together.
template <class C>
__device__ void set_loop(ChainSmem<C>& sm, const AttnParams& p, uint32_t tmem, int set) {
  const int quad = (threadIdx.x >> 5) & 3;
  const int row = quad * 32 + (threadIdx.x & 31);   // query row == TMEM lane
  const uint32_t lanes = (uint32_t)(quad * 32) << 16;
  const uint32_t tO = tmem + 384 + lanes;
  const float limit = sum_limit<C>(p);
  uint32_t base0 = 0, base1 = 0, base2 = 0;   // split tiles: tiles of the CTA's earlier units in each buffer
  uint32_t mine = 0;                          // whole tiles: tiles this set has taken
  bool ok = true;
  for (uint32_t u = 0;; ++u) {
    const uint32_t qi = u % kItemQ;
    Item itm{-1, 0, 0, -1};
    if (ok) ok = waitw(&sm.abort, p, &sm.item_full[qi], ph(u / kItemQ));
    if (ok) {
      itm = sm.items[qi];
      arrive_w(&sm.item_empty[qi]);
    }
    ok = set_and(set, ok);
    if (!ok || itm.bn < 0) break;
    const int n = itm.ntiles;
    const int tasks = kTaskSplit<C> * (n - 1);    // tasks after the first tile
    const int last = n == 1 ? 0 : tasks % kSets;  // set of the unit's last task
    float m_use = 0.f, l = 0.f;
    bool row_bad = false;
    // The tile's factors: 16-bit, S c with c = scale log2(e); fp8, the S
    // warp's TileScale of the buffer (published with s_full).
    auto factors = [&](int c) -> TileScale {
      if (C::kFp8) return sm.ts[c];
      TileScale f;
      f.c = p.scale_log2;
      f.lr = 0.f;
      f.ir = 1.f;
      f.pad = 0.f;
      return f;
    };
    auto p_valid_of = [&](int j) { return j == itm.partial ? p.p_rem_k : RF_BLOCK; };
    // S of tile j: the set's first warp waits on the buffer's barrier (the
    // tile is the buffer's (base + j / 3)-th), the other three at the set's
    // named barrier, where they take no issue slots; every warp reaches it,
    // carrying the outcome.
    // (Whole tiles: a set only ever takes tiles of its own buffer, and its
    // count of them gives the phase.)
    auto buf_of = [&](int j) { return kTaskSplit<C> == 1 ? set : j % kSets; };
    auto wait_s = [&](int j) {
      const int c = buf_of(j);
      uint32_t prev;
      if (kTaskSplit<C> == 1) {
        prev = mine++;
      } else {
        prev = (c == 0 ? base0 : c == 1 ? base1 : base2) + j / kSets;
      }
      bool got = ok;
      if (got && quad == 0) got = waitw(&sm.abort, p, &sm.s_full[c], ph(prev));
      ok = set_and(set, got);
    };
    auto do_task = [&](int j, int h) {
      wait_s(j);
      if (ok) {
        const int c = buf_of(j);
        const uint32_t tS = tmem + 128 * c + lanes;
        tc_fence_after();
        const TileScale f = factors(c);
        float hs;
        if (kTaskSplit<C> == 2) {
          hs = half_softmax<C>(tS, h, p_valid_of(j), f.c, f.lr - m_use);
          tmem_wait_st();
        } else {
          hs = tile_softmax<C>(tS, p_valid_of(j), f.c, f.lr - m_use);
        }
        row_bad |= !(hs <= limit);
        l += hs * f.ir;
        tc_fence_before();
        arrive_w(&sm.p_full[c]);
      }
    };
    if (set == 0) {
      // the unit's maximum: the row maximum of its first tile
      const uint32_t tS0 = tmem + lanes;
      wait_s(0);
      TileScale f0{};
      if (ok) {
        tc_fence_after();
        f0 = factors(0);
        m_use = tile_max(tS0, p_valid_of(0)) * f0.c;
      }
      if (ok && u >= 1) ok = waitw(&sm.abort, p, &sm.m_empty, ph(u - 1));
      if (ok) {
        sm.m_sh[row] = m_use;
        __threadfence_block();
        arrive_w(&sm.m_full);
        arrive_w(&sm.m_empty);
        // the first tile's P (its S is still in place); it stands for all
        // of the tile's tasks' arrivals
        const float ts = tile_softmax<C>(tS0, p_valid_of(0), f0.c, f0.lr - m_use);
        row_bad |= !(ts <= limit);
        l += ts * f0.ir;
        tc_fence_before();
        for (int a = 0; a < kTaskSplit<C>; ++a) arrive_w(&sm.p_full[0]);
      }
    } else {
      if (ok) ok = waitw(&sm.abort, p, &sm.m_full, ph(u));
      if (ok) {
        m_use = sm.m_sh[row];
        arrive_w(&sm.m_empty);
      }
    }
    for (int t = (set + kSets - 1) % kSets; t < tasks; t += kSets)
      do_task(1 + t / kTaskSplit<C>, t % kTaskSplit<C>);
    base0 += (n + 2) / 3;
    base1 += (n + 1) / 3;
    base2 += n / 3;
    // post this set's row sums (NaN marks a row that needs the second pass)
    if (ok && u >= 1) ok = waitw(&sm.abort, p, &sm.l_empty, ph(u - 1));
    if (ok) {
      sm.l_sh[set][row] = row_bad ? CUDART_NAN_F : l;
      __threadfence_block();
      arrive_w(&sm.l_full);
    }
    ok = set_and(set, ok);
    if (!ok) break;
    if (set != last) continue;

    // output of the unit: O / (l_0 + l_1 + l_2) (fp8: times the head's largest V scale)
    float lt = 0.f;
    ok = waitw(&sm.abort, p, &sm.l_full, ph(u));
    if (ok) {
      lt = (sm.l_sh[0][row] + sm.l_sh[1][row]) + sm.l_sh[2][row];
      arrive_w(&sm.l_empty);
    }
    const bool unit_bad = set_or(set, !(lt > 0.f && lt < CUDART_INF_F));
    ok = set_and(set, ok);
    if (!ok) break;
    ok = waitw(&sm.abort, p, &sm.o_full, ph(u));
    if (ok) {
      tc_fence_after();
      const float rl = (C::kFp8 ? p.vmax[itm.bn] : 1.f) / lt;
      uint16_t* dst = unit_bad ? nullptr : out_row<C>(p, itm.bn, itm.qt, row);
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
      if (unit_bad && quad == 0 && (threadIdx.x & 31) == 0) {
        const int slot = atomicAdd(&p.redo[1], 1);
        p.redo[2 + slot] = itm.bn * p.g.n_tiles + itm.qt;
      }
      // The next unit's first P V overwrites O only after this arrival.
      tc_fence_before();
      arrive_w(&sm.o_free);
    }
    ok = set_and(set, ok);
    if (!ok) break;
  }
}

template <class C>
__global__ void __launch_bounds__(kCThreads, 1)
    chain_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                 const __grid_constant__ CUtensorMap tm_v, const AttnParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // The struct fills the 227 KB a CTA may have, so its 1024-aligned tiles
  // cannot be aligned by hand.  Dynamic shared memory starts 1024-aligned;
  // should it not, every unit goes to the second pass.
  if (smem_u32(smem_raw) & 1023u) {
    if (blockIdx.x == 0 && threadIdx.x == 0) p.redo[1] = -1;
    return;
  }
  ChainSmem<C>& sm = *reinterpret_cast<ChainSmem<C>*>(smem_raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    using CS = ChainShape<C>;
    for (int i = 0; i < CS::kQBufs; ++i) {
      mbar_init(&sm.q_full[i], 1);
      mbar_init(&sm.q_empty[i], 1);
    }
    for (int i = 0; i < CS::kKRing; ++i) {
      mbar_init(&sm.k_full[i], 1);
      mbar_init(&sm.k_empty[i], 1);
    }
    for (int i = 0; i < CS::kVRing; ++i) {
      mbar_init(&sm.v_full[i], 1);
      mbar_init(&sm.v_empty[i], 1);
    }
    for (int i = 0; i < kSets; ++i) {
      mbar_init(&sm.s_full[i], C::kFp8 ? 2 : 1);
      mbar_init(&sm.p_full[i], 4 * kTaskSplit<C>);
      mbar_init(&sm.pv_done[i], 1);
    }
    mbar_init(&sm.o_full, 1);
    mbar_init(&sm.o_free, 4);
    mbar_init(&sm.m_full, 4);
    mbar_init(&sm.m_empty, 4 * kSets);
    mbar_init(&sm.l_full, 4 * kSets);
    mbar_init(&sm.l_empty, 4);
    for (int i = 0; i < kItemQ; ++i) {
      mbar_init(&sm.item_full[i], 1);
      mbar_init(&sm.item_empty[i], kItemReaders);
    }
    mbar_init(&sm.drain[0], 1);
    mbar_init(&sm.drain[1], 1);
    sm.abort = 0;
    fence_mbar_init();
  }
  if (warp == kWarpKProd && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  if (warp == kWarpQK) {
    tmem_alloc(&sm.tmem_base, kCTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;

  if (warp < 4 * kSets) {
    set_loop<C>(sm, p, tmem, warp >> 2);
  } else if (warp == kWarpKProd) {
    if (lane == 0) kprod_loop<C>(sm, p, &tm_q, &tm_k);
  } else if (warp == kWarpVProd) {
    if (lane == 0) vprod_loop<C>(sm, p, &tm_v);
  } else if (warp == kWarpPV) {
    pv_loop<C>(sm, p, tmem);
  } else {
    qk_loop<C>(sm, p, tmem);
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kWarpQK) tmem_dealloc(tmem, kCTmemCols);
}

// Keys and values follow the query plan (no geometry of their own).
int same_plan(const rf_plan_t& g, const rf_plan_t& gk) { return std::memcmp(&g, &gk, sizeof(rf_plan_t)) == 0; }

template <class C>
cudaError_t launch_chain_cfg(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                             const AttnParams& p, cudaStream_t stream) {
  int sms = 0;
  cudaError_t e = sm_count(&sms);
  if (e != cudaSuccess) return e;
  const size_t smem = sizeof(ChainSmem<C>);
  e = cudaFuncSetAttribute(chain_kernel<C>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  e = cudaMemsetAsync(p.counter, 0, sizeof(int), stream);
  if (e != cudaSuccess) return e;
  const int grid = std::min(sms, p.total_items);
  chain_kernel<C><<<grid, kCThreads, smem, stream>>>(tq, tk, tv, p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attention(const void* q_int, const void* k_int, const void* v_int, const uint32_t* mask,
                             int dtype, int layout, int B, int S, int N, const rf_plan_t& g, const rf_plan_t& gk,
                             float scale, void* out, int* counter, int* status, int* redo, const AttnDebug& dbg,
                             cudaStream_t stream) {
  // The redo list starts empty; the chain kernel appends, the second pass
  // (attn_kernel in list mode) takes what it lists.
  cudaError_t e = cudaMemsetAsync(redo, 0, 2 * sizeof(int), stream);
  if (e != cudaSuccess) return e;
  if (dbg.path == 1) return launch_attention_slots(q_int, k_int, v_int, mask, dtype, layout, B, S, N, g, gk, scale,
                                                   out, counter, status, redo, 0, dbg, stream);
  const uint64_t rows_q = (uint64_t)B * N * g.S_int, rows_k = (uint64_t)B * N * gk.S_int;
  const bool f16 = dtype == RF_F16;
  const CUtensorMapDataType type = f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  CUtensorMap tq, tk, tv;
  if (!make_tile_map(&tq, q_int, rows_q, type, 2) || !make_tile_map(&tk, k_int, rows_k, type, 2) ||
      !make_tile_map(&tv, v_int, rows_k, type, 2))
    return cudaErrorInvalidValue;
  AttnParams p = make_params(mask, layout, B, S, N, g, gk, scale, out, counter, status, redo, dbg);
  p.own_first = same_plan(g, gk);
  e = f16 ? launch_chain_cfg<Cfg<true, false>>(tq, tk, tv, p, stream)
          : launch_chain_cfg<Cfg<false, false>>(tq, tk, tv, p, stream);
  if (e != cudaSuccess) return e;
  AttnDebug second = dbg;
  second.skip_first_q = 0;
  return launch_attention_slots(q_int, k_int, v_int, mask, dtype, layout, B, S, N, g, gk, scale, out, counter, status,
                                redo, 1, second, stream);
}

cudaError_t launch_attention_fp8(const uint8_t* q8, const uint8_t* k8, const uint8_t* v8, const float* scales,
                                 const float* vmax, const uint32_t* mask, int dtype, int layout, int B, int S, int N,
                                 const rf_plan_t& g, const rf_plan_t& gk, float scale, void* out, int* counter,
                                 int* status, int* redo, const AttnDebug& dbg, cudaStream_t stream) {
  cudaError_t e = cudaMemsetAsync(redo, 0, 2 * sizeof(int), stream);
  if (e != cudaSuccess) return e;
  if (dbg.path == 1)
    return launch_attention_fp8_slots(q8, k8, v8, scales, vmax, mask, dtype, layout, B, S, N, g, gk, scale, out,
                                      counter, status, redo, 0, dbg, stream);
  const uint64_t rows_q = (uint64_t)B * N * g.S_int, rows_k = (uint64_t)B * N * gk.S_int;
  CUtensorMap tq, tk, tv;
  if (!make_tile_map(&tq, q8, rows_q, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1) ||
      !make_tile_map(&tk, k8, rows_k, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1) ||
      !make_tile_map(&tv, v8, rows_k, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1))
    return cudaErrorInvalidValue;
  AttnParams p = make_params(mask, layout, B, S, N, g, gk, scale, out, counter, status, redo, dbg);
  p.scales = scales;
  p.vmax = vmax;
  p.own_first = same_plan(g, gk);
  e = dtype == RF_F16 ? launch_chain_cfg<Cfg<true, true>>(tq, tk, tv, p, stream)
                      : launch_chain_cfg<Cfg<false, true>>(tq, tk, tv, p, stream);
  if (e != cudaSuccess) return e;
  AttnDebug second = dbg;
  second.skip_first_q = 0;
  return launch_attention_fp8_slots(q8, k8, v8, scales, vmax, mask, dtype, layout, B, S, N, g, gk, scale, out,
                                    counter, status, redo, 1, second, stream);
}

}  // namespace rf
