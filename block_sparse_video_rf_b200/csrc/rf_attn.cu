// Block-sparse flash attention on sm_100a tensor cores (K3), two query
// tiles per CTA, with a running maximum that is raised (and O and l
// rescaled) when a tile needs it: the second pass of every precision (the
// units chain_kernel hands back, see rf_attn_chain.cu), and the whole of K3
// when a test selects it (rf_debug_set_path).
//
// vllm-omni "RainFusion Attention", intro: prefix rows and first-frame
// blocks stay dense; every other query block attends to its highest-scoring
// key blocks.  Keys and values may have a geometry of their own
// (lite_boost.ops.sparse_attention, latent_shape_k): query tiles follow the
// query plan, KV tiles the key plan.  Persistent CTAs (one per SM) take
// units from a global counter in (head, tile) order, dense tiles of a head
// first, so the heads in flight keep their K/V in L2; in list mode they take
// the units listed by chain_kernel instead.
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
#include "rf_attn_common.cuh"

namespace rf {

namespace {

constexpr int kThreads = 384;
constexpr int kSlots = 2;
constexpr int kSlotWarps = 4;                            // softmax warps per slot
constexpr uint32_t kRegsSoftmax = 216, kRegsControl = 64;
constexpr uint32_t kTmemCols = 512;

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

// ---------------------------------------------------------------- producer
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
    const int w = atomicAdd(p.list_mode ? &p.redo[0] : p.counter, 1);
    const uint32_t it = c & 1;
    if (c >= 2 && !wait1(&sm.abort, p, &sl.item_empty[it], ph((c >> 1) - 1))) {
      ok = false;
      break;
    }
    const uint32_t* mrow;
    const Item itm = make_item(p, unit_of(p, w), mrow);
    sl.items[it] = itm;
    mbar_arrive(&sl.item_full[it]);
    if (itm.bn < 0) break;

    const int base = itm.bn * S_int_k;   // the unit's KV rows
    const float* sc_k = C::kFp8 ? p.scales + (size_t)BN * p.g.n_tiles + (size_t)itm.bn * p.gk.n_tiles : nullptr;
    const float* sc_v = C::kFp8 ? sc_k + (size_t)BN * p.gk.n_tiles : nullptr;
    if (c >= 1 && !wait1(&sm.abort, p, &sl.q_empty, ph(c - 1))) {
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
      if (ku >= 1 && !wait1(&sm.abort, p, &sl.k_empty[ks], ph(ku - 1))) {
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
      if (vu >= 1 && !wait1(&sm.abort, p, &sl.v_empty[vs], ph(vu - 1))) {
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
  load_scores<4>(tS, p_valid, s);
  float alpha = 1.f;
  bool rescale = false;
  float tsum;
  if (first) {
    m_use = row_max<4>(s) * c;
    tsum = exp_scores<C, 4>(s, c, lr - m_use, p_valid, pk);
  } else {
    tsum = exp_scores<C, 4>(s, c, lr - m_use, p_valid, pk);
    if (__any_sync(0xFFFFFFFFu, !(tsum <= kSumLimit))) {
      load_scores<4>(tS, p_valid, s);
      const float mx_s = row_max<4>(s) * c;
      if (mx_s > m_use + kRescaleThreshold) {
        alpha = ex2_approx(m_use - mx_s);
        m_use = mx_s;
        rescale = true;
      }
      tsum = exp_scores<C, 4>(s, c, lr - m_use, p_valid, pk);
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
    if (!waitw(&sm.abort, p, &sl.k_full[ks], ph(tt / C::kKStages))) return false;
    // read before the MMAs: once they finish, the producer may refill the stage
    const float sk = C::kFp8 ? sl.kv_scale[ks][0] : 0.f, sv = C::kFp8 ? sl.kv_scale[ks][1] : 0.f;
    if (tt >= 1 && !waitw(&sm.abort, p, &sl.pv_done, ph(tt - 1))) return false;
    tc_fence_after();
    issue_qk<C>(s_tmem, q_lo, k_lo0 + ks * (C::kTileBytes >> 4), hi);
    mma_commit_elect(&sl.s_full);
    mma_commit_elect(&sl.k_empty[ks]);
    if (last_of_unit) mma_commit_elect(&sl.q_empty);
    issued = true;
    if ((threadIdx.x & 31) == 0) {
      if (C::kFp8) sl.ts[tt & 1] = tile_scale(p, q_scale, sk, sv, unit_vmax);
      mbar_arrive(&sl.s_full);
    }
    __syncwarp();
    return true;
  };

  for (;; ++c) {
    // Every warp of the slot reaches every rendezvous: a warp whose wait
    // failed carries ok = false to the next one, where all four leave.
    const uint32_t it = c & 1;
    Item itm{-1, 0, 0, -1};
    if (ok) ok = waitw(&sm.abort, p, &sl.item_full[it], ph(c >> 1));
    if (ok) {
      itm = sl.items[it];
      arrive_w(&sl.item_empty[it]);
    }
    ok = slot_vote(bar_id, ok);
    if (!ok || itm.bn < 0) break;
    if (issuer) {
      ok = waitw(&sm.abort, p, &sl.q_full, ph(c));
      if (C::kFp8 && ok) {
        q_scale = sl.q_scale;
        unit_vmax = p.vmax[itm.bn];
      }
      if (ok) ok = qk(t, itm.ntiles == 1);
    }
    const float out_scale = C::kFp8 ? p.vmax[itm.bn] : 1.f;

    float m_use = -CUDART_INF_F, l = 0.f;
    for (int j = 0; j < itm.ntiles; ++j, ++t) {
      if (ok) ok = waitw(&sm.abort, p, &sl.s_full, ph(t));
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
        ok = waitw(&sm.abort, p, &sl.v_full[vs], ph(t / C::kVStages));
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
    if (ok) ok = waitw(&sm.abort, p, &sl.pv_done, ph(t - 1));
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
  // second pass with nothing listed: leave before any setup
  if (p.list_mode && p.redo[1] == 0) return;
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
template <class C>
cudaError_t launch_cfg(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const AttnParams& p,
                       cudaStream_t stream) {
  int sms = 0;
  cudaError_t e = sm_count(&sms);
  if (e != cudaSuccess) return e;
  const size_t smem = sizeof(Smem<C>) + 1024;
  e = cudaFuncSetAttribute(attn_kernel<C>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  if (!p.list_mode) {
    e = cudaMemsetAsync(p.counter, 0, sizeof(int), stream);
    if (e != cudaSuccess) return e;
  }
  const int grid = std::min(sms, p.total_items);
  attn_kernel<C><<<grid, kThreads, smem, stream>>>(tq, tk, tv, p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attention_slots(const void* q_int, const void* k_int, const void* v_int, const uint32_t* mask,
                                   int dtype, int layout, int B, int S, int N, const rf_plan_t& g,
                                   const rf_plan_t& gk, float scale, void* out, int* counter, int* status, int* redo,
                                   int list_mode, const AttnDebug& dbg, cudaStream_t stream) {
  const uint64_t rows_q = (uint64_t)B * N * g.S_int, rows_k = (uint64_t)B * N * gk.S_int;
  const bool f16 = dtype == RF_F16;
  const CUtensorMapDataType type = f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  CUtensorMap tq, tk, tv;
  if (!make_tile_map(&tq, q_int, rows_q, type, 2) || !make_tile_map(&tk, k_int, rows_k, type, 2) ||
      !make_tile_map(&tv, v_int, rows_k, type, 2))
    return cudaErrorInvalidValue;
  AttnParams p = make_params(mask, layout, B, S, N, g, gk, scale, out, counter, status, redo, dbg);
  p.list_mode = list_mode;
  return f16 ? launch_cfg<Cfg<true, false>>(tq, tk, tv, p, stream)
             : launch_cfg<Cfg<false, false>>(tq, tk, tv, p, stream);
}

cudaError_t launch_attention_fp8_slots(const uint8_t* q8, const uint8_t* k8, const uint8_t* v8, const float* scales,
                                       const float* vmax, const uint32_t* mask, int dtype, int layout, int B, int S,
                                       int N, const rf_plan_t& g, const rf_plan_t& gk, float scale, void* out,
                                       int* counter, int* status, int* redo, int list_mode, const AttnDebug& dbg,
                                       cudaStream_t stream) {
  const uint64_t rows_q = (uint64_t)B * N * g.S_int, rows_k = (uint64_t)B * N * gk.S_int;
  CUtensorMap tq, tk, tv;
  if (!make_tile_map(&tq, q8, rows_q, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1) ||
      !make_tile_map(&tk, k8, rows_k, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1) ||
      !make_tile_map(&tv, v8, rows_k, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1))
    return cudaErrorInvalidValue;
  AttnParams p = make_params(mask, layout, B, S, N, g, gk, scale, out, counter, status, redo, dbg);
  p.scales = scales;
  p.vmax = vmax;
  p.list_mode = list_mode;
  return dtype == RF_F16 ? launch_cfg<Cfg<true, true>>(tq, tk, tv, p, stream)
                         : launch_cfg<Cfg<false, true>>(tq, tk, tv, p, stream);
}

}  // namespace rf
