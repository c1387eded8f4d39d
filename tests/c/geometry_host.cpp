// Host check of the block fast path of the reorder geometry: for every
// sparse block of many plans, rf_src_in_block over rf_block_tiles gives the
// same token as rf_src_of_row for each of the block's 128 rows.  Prints the
// number of rows compared; returns non-zero on the first mismatch.
#include <cstdio>

#include "rf_geometry.h"

extern "C" rf_status_t rf_plan(int S, int txt_len, int T, int H, int W, int block_size, float sparsity, rf_plan_t* out);

int main() {
  const int grids[][4] = {{0, 62, 24, 42},  {256, 62, 24, 42}, {37, 8, 21, 43}, {19, 5, 24, 40}, {0, 21, 45, 80},
                          {512, 8, 48, 64}, {0, 4, 32, 32},    {7, 3, 16, 16},  {0, 128, 64, 64}, {3, 9, 17, 31},
                          {0, 2, 8, 8},     {11, 33, 40, 24},  {0, 1, 64, 64},  {5, 7, 9, 130}};
  long rows = 0;
  for (const auto& gr : grids) {
    rf_plan_t g;
    const int S = gr[0] + gr[1] * gr[2] * gr[3];
    if (rf_plan(S, gr[0], gr[1], gr[2], gr[3], RF_BLOCK, 0.5f, &g) != RF_OK) {
      std::printf("plan refused: %d %d %d %d\n", gr[0], gr[1], gr[2], gr[3]);
      return 2;
    }
    if (g.dense) continue;
    for (int blk = 0; blk < g.nb; ++blk) {
      const RfBlockTiles b = rf_block_tiles(g, blk);
      for (int r = 0; r < RF_BLOCK; ++r, ++rows) {
        const int want = rf_src_of_row(g, g.P_pad + blk * RF_BLOCK + r), got = rf_src_in_block(g, b, r);
        if (want != got) {
          std::printf("mismatch: grid %d %d %d %d block %d row %d: %d against %d\n", gr[0], gr[1], gr[2], gr[3], blk,
                      r, got, want);
          return 1;
        }
      }
    }
  }
  std::printf("%ld rows agree\n", rows);
  return 0;
}
