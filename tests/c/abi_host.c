/* A plain C11 caller of the library's host-only entry points: the header
 * compiles as C, the library links, and the geometry plan of the MiniMax-H3
 * 1344x768 grid gives the worked numbers of the vllm-omni "RainFusion
 * Attention" page, "Geometry handling" (62,496 video rows, 2,976 promoted,
 * 465 sparse blocks of 128).  No CUDA call is made: every entry point used
 * here validates and plans on the host, or refuses its arguments before
 * touching the GPU.  Prints one line per check and returns non-zero on the
 * first failure. */
#include <stdio.h>
#include <string.h>

#include "rfsa.h"

static int fails = 0;

static void check(int ok, const char* what) {
  printf("%s %s\n", ok ? "ok  " : "FAIL", what);
  if (!ok) ++fails;
}

int main(void) {
  rf_plan_t p;
  memset(&p, 0, sizeof(p));
  rf_status_t st = rf_plan(256 + 62 * 24 * 42, 256, 62, 24, 42, 128, 0.8f, &p);
  check(st == RF_OK, "rf_plan accepts the MiniMax-H3 geometry");
  check(p.T * p.H * p.W == 62496, "62,496 video rows");
  check(p.n_promoted + p.n_tail == 2976, "2,976 promoted rows");
  check(p.nb == 465 && p.nb * RF_BLOCK == 59520, "465 sparse blocks of 128 (59,520 rows)");
  check(p.ff == 8 && p.k == 93 && !p.dense, "8 first-frame blocks, k = 93 at sparsity 0.8");

  rf_ws_layout_t lay;
  st = rf_workspace_layout(1, 56, RF_HEAD_DIM, &p, &lay);
  check(st == RF_OK && lay.total == rf_workspace_size(1, p.S, 56, 128, 256, 62, 24, 42),
        "workspace layout and size agree");
  check(lay.q_int % 256 == 0 && lay.mask % 256 == 0 && lay.redo % 256 == 0, "workspace regions 256-byte aligned");

  /* argument errors come back before any CUDA call, with a reason */
  st = rf_plan(4096, 0, 4, 32, 32, 128, 1.5f, &p);
  check(st == RF_ERR_ARG && strlen(rf_last_error_string()) > 0, "sparsity 1.5 is RF_ERR_ARG, with a message");
  st = rf_plan(4096, 0, 4, 32, 32, 64, 0.5f, &p);
  check(st == RF_ERR_UNSUPPORTED, "block_size 64 is RF_ERR_UNSUPPORTED");
  st = rf_sparse_attention((const void*)0x1000, (const void*)0x1000, (const void*)0x1000, (rf_layout_t)7, 1, 4096, 2,
                           128, 0, 4, 32, 32, 128, 0.5f, 0.f, (void*)0x2000, NULL);
  check(st == RF_ERR_LAYOUT, "an unknown layout is RF_ERR_LAYOUT");
  st = rf_sparse_attention((const void*)0x1008, (const void*)0x1000, (const void*)0x1000, RF_BSND, 1, 4096, 2, 128,
                           0, 4, 32, 32, 128, 0.5f, 0.f, (void*)0x2000, NULL);
  check(st == RF_ERR_ARG, "a q pointer off a 16-byte boundary is RF_ERR_ARG");

  /* the host-buffer call of any type, precision and key geometry refuses its
   * arguments before it copies anything */
  static char hbuf[64];
  st = rf_sparse_attention_host_ex(hbuf, hbuf, hbuf, (rf_dtype_t)5, RF_PREC_NATIVE, RF_BSND, 1, 4096, 2, 128, 0, 4,
                                   32, 32, 0, 0, 0, 0, 128, 0.5f, 0.f, hbuf, NULL);
  check(st == RF_ERR_ARG, "host call: an unknown input type is RF_ERR_ARG");
  st = rf_sparse_attention_host_ex(hbuf, NULL, hbuf, RF_F16, RF_PREC_FP8, RF_BSND, 1, 4096, 2, 128, 0, 4, 32, 32, 0,
                                   0, 0, 0, 128, 0.5f, 0.f, hbuf, NULL);
  check(st == RF_ERR_ARG, "host call: a NULL host buffer is RF_ERR_ARG");
  st = rf_sparse_attention_host_ex(hbuf, hbuf, hbuf, RF_BF16, RF_PREC_NATIVE, RF_BNSD, 1, 4096, 2, 128, 0, 4, 32, 32,
                                   5000, 5, 32, 32, 128, 0.5f, 0.f, hbuf, NULL);
  check(st == RF_ERR_ARG, "host call: S_kv other than txt_len + t h w is RF_ERR_ARG");
  return fails ? 1 : 0;
}
