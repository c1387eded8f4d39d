// Geometry of the rf_v2 token reorder, usable from host and device code.
//
// vllm-omni "RainFusion Attention", "Geometry handling": video tokens are
// rearranged into 8x8 spatial tiles; tokens outside the 8x8-aligned grid of
// each frame are promoted to the always-kept prefix (no padding of the
// video).  Intro: tokens in (t, h, w) order, 128-token blocks, first-frame
// blocks and prefix rows stay dense, fewer than 32 blocks falls back to
// dense.  lite_boost.ops.sparse_attention, txt_len: text rows stay in front
// and are not reordered.
//
// Internal row order of one (b, head), r in [0, S_int):
//   [0, txt_len)                         text tokens
//   [txt_len, txt_len + n_promoted)      non-aligned video tokens, (t, y, x) order
//   [.., P)                              aligned tokens past the last whole block
//   [P, P_pad)                           zero rows (never read as keys, never written out)
//   [P_pad, P_pad + 128 nb)              sparse blocks: position s of the aligned
//                                        order = frame, tile row, tile column,
//                                        row in tile, column in tile
// In the dense fallback the prefix is the whole sequence in its own order.
#pragma once

#include <stdint.h>

#include "rfsa.h"

#ifdef __CUDACC__
#define RF_HD __host__ __device__ __forceinline__
#else
#define RF_HD inline
#endif

// Aligned-order position s (0 <= s < T*Ha*Wa) -> sequence index of the token.
RF_HD int rf_src_of_aligned(const rf_plan_t& g, int s) {
  const int tiles_x = g.Wa >> 3;
  const int tiles_per_frame = (g.Ha >> 3) * tiles_x;
  const int tile = s >> 6, in_tile = s & 63;
  const int t = tile / tiles_per_frame, tf = tile - t * tiles_per_frame;
  const int ty = tf / tiles_x, tx = tf - ty * tiles_x;
  const int y = (ty << 3) + (in_tile >> 3), x = (tx << 3) + (in_tile & 7);
  return g.txt_len + (t * g.H + y) * g.W + x;
}

// A sparse block is two consecutive 8x8 tiles of the aligned order (tiles
// 2 blk and 2 blk + 1): their frames and top-left corners, with two
// divisions for the block instead of two per row.
struct RfBlockTiles {
  int t[2], y[2], x[2];
};
RF_HD RfBlockTiles rf_block_tiles(const rf_plan_t& g, int blk) {
  const int tiles_x = g.Wa >> 3, tiles_y = g.Ha >> 3;
  const int tiles_per_frame = tiles_y * tiles_x;
  const int tile = 2 * blk;
  int t = tile / tiles_per_frame;
  const int tf = tile - t * tiles_per_frame;
  int ty = tf / tiles_x, tx = tf - ty * tiles_x;
  RfBlockTiles b;
  b.t[0] = t, b.y[0] = ty << 3, b.x[0] = tx << 3;
  if (++tx == tiles_x) {   // the next tile: the next column, row or frame
    tx = 0;
    if (++ty == tiles_y) ty = 0, ++t;
  }
  b.t[1] = t, b.y[1] = ty << 3, b.x[1] = tx << 3;
  return b;
}
// Sequence index of row r (0 <= r < 128) of that block: the same as
// rf_src_of_aligned(g, 128 blk + r).
RF_HD int rf_src_in_block(const rf_plan_t& g, const RfBlockTiles& b, int r) {
  const int h = r >> 6, in_tile = r & 63;
  return g.txt_len + (b.t[h] * g.H + b.y[h] + (in_tile >> 3)) * g.W + b.x[h] + (in_tile & 7);
}

// Internal row r -> sequence index of its token, or -1 for a pad row.
RF_HD int rf_src_of_row(const rf_plan_t& g, int r) {
  if (r < g.P) {
    if (g.dense || r < g.txt_len) return r;
    int p = r - g.txt_len;
    if (p < g.n_promoted) {
      const int per_frame = g.H * g.W - g.Ha * g.Wa;
      const int t = p / per_frame, q = p - t * per_frame;
      const int right = g.W - g.Wa;           // non-aligned columns of each aligned row
      int y, x;
      if (q < g.Ha * right) {
        y = q / right;
        x = g.Wa + (q - y * right);
      } else {
        const int q2 = q - g.Ha * right;
        y = g.Ha + q2 / g.W;
        x = q2 - (y - g.Ha) * g.W;
      }
      return g.txt_len + (t * g.H + y) * g.W + x;
    }
    return rf_src_of_aligned(g, g.nb * RF_BLOCK + (p - g.n_promoted));
  }
  if (r < g.P_pad) return -1;
  return rf_src_of_aligned(g, r - g.P_pad);
}

// Element offset of token s of head (b, n) in the caller's layout.
RF_HD int64_t rf_token_offset(int layout, int B, int S, int N, int b, int n, int s) {
  (void)B;
  if (layout == RF_BSND) return ((int64_t)(b * (int64_t)S + s) * N + n) * RF_HEAD_DIM;
  return ((int64_t)(b * (int64_t)N + n) * S + s) * RF_HEAD_DIM;
}
