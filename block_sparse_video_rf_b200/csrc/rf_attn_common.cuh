// Pieces shared by the two block-sparse attention kernels (K3):
// attn_kernel (rf_attn.cu: two query tiles per CTA; the fp8 path and the
// pass that redoes the units the other kernel hands back) and chain_kernel
// (rf_attn_chain.cu: one query tile per CTA, three tiles of keys in flight;
// the 16-bit path).
//
// lite_boost.ops.sparse_attention, rf_v2 pipeline: rain_fusion_attention
// over the kept KV blocks, then the inverse reorder (fused here: each output
// row is written straight to its token's place in the caller's layout).
// Work unit: one 128-row query tile of one (b, head).  Its KV list is every
// key prefix tile, then either every key block (dense tile) or the blocks
// set in its mask row, in ascending order.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math_constants.h>

#include <algorithm>

#include "rf_dtype.h"
#include "rf_geometry.h"
#include "rf_kernels.h"
#include "sm100_ptx.cuh"

namespace rf {

namespace {

constexpr int kBoxBytes = RF_BLOCK * 128;                // one TMA box: 128 rows x 128 bytes
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
  // (the rest on MUFU): measured best split for each path (16-bit, under the power cap)
  static constexpr int kPolyEvery = kFp8 ? 3 : 8;
  static constexpr uint32_t kIdescQK =
      kFp8 ? make_idesc_e4m3(128, 128, false) : make_idesc_f16kind(128, 128, false, !kF16);
  static constexpr uint32_t kIdescPV =
      kFp8 ? make_idesc_e4m3(128, 128, false) : make_idesc_f16kind(128, 128, true, !kF16);
};

struct Item {
  int bn, qt, ntiles;
  int partial;   // chain_kernel: place of the partial key prefix tile in the unit's tile order (-1: none)
};

// Per-tile factors of the fp8 path, written by the slot's issuer before its
// arrival on s_full: c = scale * log2(e) * sq * sk (multiplies S), lr =
// log2(sv / vmax) (added to P's exponent), ir = vmax / sv (l adds P's sum
// times ir).
struct TileScale {
  float c, lr, ir, pad;
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
  // Units handed from chain_kernel to attn_kernel: [0] the second pass's work
  // counter, [1] the number of units listed (-1: every unit), [2 ...] their ids.
  int* redo;
  int list_mode;            // attn_kernel: take units from `redo` instead of all of them
  int own_first;            // chain_kernel: keys share the query plan, so a unit starts with its own key tile
  float sum_limit;          // chain_kernel: tile sum of P that sends a unit to the second pass (0: the type's)
  uint64_t wait_limit_ns;   // limit of every device-side wait
  int skip_first_q;         // test control: the first unit's Q load is never issued
};

// The fp8 factors of one tile from the unit's Q block scale sq, the tile's
// K and V block scales sk, sv and the head's largest V block scale vmax.
__device__ __forceinline__ TileScale tile_scale(const AttnParams& p, float sq, float sk, float sv, float vmax) {
  TileScale f;
  f.c = p.scale_log2 * sq * sk;
  const bool use_r = sv > 0.f && vmax > 0.f;   // an all-zero V block adds nothing whatever P is
  f.lr = use_r ? __log2f(sv / vmax) : 0.f;
  f.ir = use_r ? vmax / sv : 1.f;
  f.pad = 0.f;
  return f;
}

__device__ __forceinline__ bool is_dense_tile(const AttnParams& p, int qt) {
  return p.g.dense || qt < p.n_ptiles || (qt - p.n_ptiles) < p.g.ff;
}

// Unit id of work item w, or -1 past the end.
__device__ __forceinline__ int unit_of(const AttnParams& p, int w) {
  if (!p.list_mode) return w < p.total_items ? w : -1;
  const int n = p.redo[1];
  if (n < 0) return w < p.total_items ? w : -1;
  return w < n ? p.redo[2 + w] : -1;
}

// The unit of work item w: its (head, query tile) and KV tile count; `mrow`
// is its mask row (nullptr for a dense tile).
__device__ __forceinline__ Item make_item(const AttnParams& p, int unit, const uint32_t*& mrow) {
  Item itm{-1, 0, 0, -1};
  mrow = nullptr;
  if (unit < 0) return itm;
  itm.bn = unit / p.g.n_tiles;
  itm.qt = unit - itm.bn * p.g.n_tiles;
  if (is_dense_tile(p, itm.qt)) {
    itm.ntiles = p.gk.n_tiles;
  } else {
    mrow = p.mask + ((size_t)itm.bn * p.g.nb + (itm.qt - p.n_ptiles)) * p.gk.mask_words;
    int cnt = 0;
    for (int wd = 0; wd < p.gk.mask_words; ++wd) cnt += __popc(mrow[wd]);
    itm.ntiles = p.n_ptiles_k + cnt;
  }
  return itm;
}

// Bounded wait by one thread (see rf_wait).
__device__ __forceinline__ bool wait1(volatile int* abort, const AttnParams& p, uint64_t* bar, uint32_t parity) {
  return rf_wait(bar, parity, abort, p.status, RF_ERR_TIMEOUT, p.wait_limit_ns);
}
// Bounded wait by a whole warp, with a warp-uniform outcome (the warp then
// runs .sync.aligned tcgen05 instructions together or leaves together).
__device__ __forceinline__ bool waitw(volatile int* abort, const AttnParams& p, uint64_t* bar, uint32_t parity) {
  return __all_sync(0xFFFFFFFFu, wait1(abort, p, bar, parity));
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

// Visits the KV tile rows of one unit in order: every prefix tile, then every
// sparse block (dense unit) or the set bits of its mask row.  With own >= 0
// (a key tile index: prefix tile, or n_ptiles + block) that tile comes
// first and the rest follow in that order.
struct KvIter {
  int base, n_ptiles, nb, words;
  const uint32_t* mrow;   // nullptr for a dense unit
  int t, wd;
  uint32_t bits;
  int own;                // the tile visited first, or -1
  bool own_done;
  __device__ void init(int base_, const AttnParams& p, const uint32_t* mrow_, int own_ = -1) {
    base = base_;
    n_ptiles = p.n_ptiles_k;
    nb = p.gk.nb;
    words = p.gk.mask_words;
    mrow = mrow_;
    t = 0;
    wd = 0;
    bits = 0;
    own = own_;
    own_done = own_ < 0;
  }
  // Row of the next KV tile, or -1 at the end.
  __device__ int next() {
    if (!own_done) {
      own_done = true;
      return base + own * RF_BLOCK;
    }
    int r;
    do {
      r = next_natural();
    } while (own >= 0 && r == base + own * RF_BLOCK);
    return r;
  }
  __device__ int next_natural() {
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

// The key tile of a unit's own rows (same index as its query tile) when keys
// share the query plan and the unit reads that tile, else -1.  Attention is
// strongest near the query in video, so the unit's reference maximum is best
// taken there.
__device__ __forceinline__ int own_tile(const AttnParams& p, const Item& itm, const uint32_t* mrow) {
  if (!p.own_first || itm.bn < 0) return -1;
  if (itm.qt < p.n_ptiles || !mrow) return itm.qt;
  const int b = itm.qt - p.n_ptiles;
  return ((mrow[b >> 5] >> (b & 31)) & 1u) ? itm.qt : -1;
}
// Place of the partial key prefix tile (index n_ptiles_k - 1) in the order
// KvIter gives with `own` first; -1 when the prefix has no partial tile.
__device__ __forceinline__ int partial_place(const AttnParams& p, int own) {
  if (p.p_rem_k == 0) return -1;
  const int part = p.n_ptiles_k - 1;
  if (own < 0 || own < part) return part;
  return own == part ? 0 : part + 1;
}

// One 128 x 128 tile: one box of 128 bytes per row (fp8) or two boxes of 64
// 16-bit columns.
template <class C>
__device__ __forceinline__ void load_tile(uint8_t* dst, const CUtensorMap* map, uint64_t* bar, int row,
                                          uint64_t policy) {
  mbar_arrive_expect_tx(bar, C::kTileBytes);
#pragma unroll
  for (int b = 0; b < C::kBoxes; ++b) tma_load_2d(dst + b * kBoxBytes, map, bar, b * 64, row, policy);
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
// keys).  P of keys 64..127 starts `half_col` columns after P of keys 0..63
// (contiguous when half_col is 8 kSteps / 2).  16-bit V is MN-major: 16 keys
// are 16 rows of 128 B further.  fp8 V is stored transposed (K-major): 32
// keys are 32 B further.
template <class C>
__device__ __forceinline__ void issue_pv(uint32_t o_tmem, uint32_t p_tmem, uint32_t v_lo, uint32_t hi,
                                         bool accumulate, uint32_t half_col = 8 * (C::kSteps / 2)) {
#pragma unroll
  for (int kk = 0; kk < C::kSteps; ++kk) {
    const uint32_t acc = (accumulate || kk > 0) ? 1u : 0u;
    const uint32_t pc = kk < C::kSteps / 2 ? kk * 8 : half_col + (kk - C::kSteps / 2) * 8;
    if (C::kFp8)
      mma_ts_lo_elect_f8(o_tmem, p_tmem + pc, v_lo + kk * 2, hi, C::kIdescPV, acc);
    else
      mma_ts_lo_elect(o_tmem, p_tmem + pc, v_lo + kk * (2048 >> 4), hi, C::kIdescPV, acc);
  }
}

// ---------------------------------------------------------------- softmax pieces
// P = 2^(s c + off) for `kQ` groups of 32 scores (already in registers),
// with their sum; writes the packed P words (16-bit: two per word; fp8:
// four).  `p_valid` counts the valid keys from the first score given; the
// rest get P = 0.  16-bit: the sum is taken over P as rounded to its type,
// the very weights P V multiplies, so the row's weights divided by l sum to
// one (the output is a weighted mean of V rows up to the fp32 sums).  fp8:
// the sum of P before rounding.
template <class C, int kQ, bool kPartial>
__device__ __forceinline__ float exp_scores_(const uint32_t (&s)[kQ][32], float c, float off, int p_valid,
                                             uint32_t (&pk)[kQ * (C::kFp8 ? 8 : 16)]) {
  constexpr int kPoly = C::kPolyEvery;
  const uint64_t c2 = f2_pack(c, c);
  const uint64_t negm = f2_pack(off, off);
  constexpr bool partial = kPartial;
  uint64_t sum2[4] = {0, 0, 0, 0};  // fp8: four packed partial sums
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};   // 16-bit: the same eight sums unpacked
  float hold0 = 0.f, hold1 = 0.f;   // fp8: the first pair of a 4-key word
#pragma unroll
  for (int q4 = 0; q4 < kQ; ++q4)
#pragma unroll
    for (int e = 0; e < 32; e += 2) {
      const int i = 16 * q4 + (e >> 1);     // pair index
      const uint64_t x2 = f2_fma(f2_pack(__uint_as_float(s[q4][e]), __uint_as_float(s[q4][e + 1])), c2, negm);
      uint64_t p2;
      if ((i % kPoly) == kPoly - 1) {
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
      float a0, a1;
      f2_unpack(p2, a0, a1);
      if (C::kFp8) {
        sum2[i & 3] = f2_add(sum2[i & 3], p2);
        if (i & 1)
          pk[i >> 1] = pack_e4m3x4(hold0, hold1, a0, a1);
        else {
          hold0 = a0;
          hold1 = a1;
        }
      } else {
        const uint32_t wd = pack_half2<C::kF16>(a0, a1);
        pk[i] = wd;
        add_half2_to<C::kF16>(wd, acc[2 * (i & 3)], acc[2 * (i & 3) + 1]);
      }
    }
  if (!C::kFp8) {
#pragma unroll
    for (int k = 0; k < 4; ++k) sum2[k] = f2_pack(acc[2 * k], acc[2 * k + 1]);
  }
  float s0, s1, s2, s3;
  f2_unpack(f2_add(sum2[0], sum2[1]), s0, s1);
  f2_unpack(f2_add(sum2[2], sum2[3]), s2, s3);
  return (s0 + s1) + (s2 + s3);
}
// The common case (every key valid) without any masking code.
template <class C, int kQ>
__device__ __forceinline__ float exp_scores(const uint32_t (&s)[kQ][32], float c, float off, int p_valid,
                                            uint32_t (&pk)[kQ * (C::kFp8 ? 8 : 16)]) {
  return p_valid >= 32 * kQ ? exp_scores_<C, kQ, false>(s, c, off, p_valid, pk)
                            : exp_scores_<C, kQ, true>(s, c, off, p_valid, pk);
}

// `kQ` groups of 32 scores from TMEM columns [col, col + 32 kQ) of the warp's
// lanes; keys at or past `p_valid` (counted from col) read as -inf.
template <int kQ>
__device__ __forceinline__ void load_scores(uint32_t tS, int p_valid, uint32_t (&s)[kQ][32]) {
#pragma unroll
  for (int q4 = 0; q4 < kQ; ++q4) tmem_ld32(tS + 32 * q4, s[q4]);
  tmem_wait_ld();
#pragma unroll
  for (int q4 = 0; q4 < kQ; ++q4) reg_fence32(s[q4]);
  if (p_valid < 32 * kQ) {
#pragma unroll
    for (int q4 = 0; q4 < kQ; ++q4)
#pragma unroll
      for (int e = 0; e < 32; ++e)
        if (32 * q4 + e >= p_valid) s[q4][e] = __float_as_uint(-CUDART_INF_F);
  }
}

template <int kQ>
__device__ __forceinline__ float row_max(const uint32_t (&s)[kQ][32]) {
  float mx8[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) mx8[i] = -CUDART_INF_F;
#pragma unroll
  for (int q4 = 0; q4 < kQ; ++q4)
#pragma unroll
    for (int e = 0; e < 32; e += 2)
      mx8[(e >> 1) & 7] = max3f(mx8[(e >> 1) & 7], __uint_as_float(s[q4][e]), __uint_as_float(s[q4][e + 1]));
  return max3f(max3f(mx8[0], mx8[1], mx8[2]), max3f(mx8[3], mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7]));
}

// Output row of query row `row` of unit (bn, qt) in the caller's layout, or
// nullptr for a padding row.
template <class C>
__device__ __forceinline__ uint16_t* out_row(const AttnParams& p, int bn, int qt, int row) {
  const int b = bn / p.N, nh = bn - b * p.N;
  const int src = rf_src_of_row(p.g, qt * RF_BLOCK + row);
  return src >= 0 ? static_cast<uint16_t*>(p.out) + rf_token_offset(p.layout, p.B, p.S, p.N, b, nh, src) : nullptr;
}

// ---------------------------------------------------------------- host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn encode_fn() {
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
inline bool make_tile_map(CUtensorMap* map, const void* base, uint64_t rows, CUtensorMapDataType type,
                          int elem_bytes) {
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

inline AttnParams make_params(const uint32_t* mask, int layout, int B, int S, int N, const rf_plan_t& g,
                              const rf_plan_t& gk, float scale, void* out, int* counter, int* status, int* redo,
                              const AttnDebug& dbg) {
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
  p.redo = redo;
  p.list_mode = 0;
  p.own_first = 0;
  p.sum_limit = dbg.sum_limit;
  p.wait_limit_ns = dbg.wait_limit_ns > 0 ? (uint64_t)dbg.wait_limit_ns : kWaitLimitNs;
  p.skip_first_q = dbg.skip_first_q;
  return p;
}

inline cudaError_t sm_count(int* sms) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  return cudaDeviceGetAttribute(sms, cudaDevAttrMultiProcessorCount, dev);
}

}  // namespace

}  // namespace rf
