// C ABI of the library: argument checks, the geometry plan, workspace
// layout, and the launch sequence K1 -> K2 -> K3 on the caller's stream.
//
// Argument rules follow lite_boost.ops.sparse_attention (input_layout must be
// BSND or BNSD; scale defaults to head_dim ** -0.5; sparsity in [0, 1];
// output shaped like q) and vllm-omni "RainFusion Attention" (sparsity finite
// in [0, 1]; 128-token blocks; fewer than 32 video blocks or no geometry is
// dense attention).
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <mutex>
#include <string>
#include <vector>

#include "rf_geometry.h"
#include "rf_kernels.h"
#include "rfsa.h"

namespace {

thread_local std::string g_last_error;

// Process-wide test controls of the attention kernel (rf_debug_set_wait).
std::mutex g_debug_mu;
rf::AttnDebug g_debug;
cudaEvent_t g_stage_event = nullptr;   // rf_debug_set_stage_event

// NVTX range around a stage's launches (host side: it marks when the work
// is enqueued).  Header-only NVTX: without a tool attached a push or pop is a
// check of one pointer.
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

rf::AttnDebug debug_settings() {
  std::lock_guard<std::mutex> lock(g_debug_mu);
  return g_debug;
}

rf_status_t fail(rf_status_t code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return code;
}

rf_status_t ok() {
  g_last_error.clear();
  return RF_OK;
}

rf_status_t cuda_fail(cudaError_t e, const char* what) {
  return fail(RF_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

struct Dims {
  int B, S, N, D;
};

rf_status_t check_common(rf_layout_t layout, int B, int S, int N, int D) {
  if (layout != RF_BSND && layout != RF_BNSD) return fail(RF_ERR_LAYOUT, "input layout must be BSND (0) or BNSD (1)");
  if (B <= 0 || S <= 0 || N <= 0) return fail(RF_ERR_ARG, "B, S and N must be positive");
  if (B > 65535 || (int64_t)B * N > 65535) return fail(RF_ERR_UNSUPPORTED, "B * N above 65535");
  if (D != RF_HEAD_DIM) return fail(RF_ERR_UNSUPPORTED, "head dim must be 128 (got %d)", D);
  return RF_OK;
}

// The kernels read and write 16-byte vectors of a token's head vector, so
// every tensor must start on a 16-byte boundary (rows are 256 bytes long).
rf_status_t check_aligned16(const void* p, const char* name) {
  if (reinterpret_cast<uintptr_t>(p) & 15) return fail(RF_ERR_ARG, "%s is not 16-byte aligned", name);
  return RF_OK;
}

rf_status_t check_types(rf_dtype_t dtype, rf_precision_t precision) {
  if (dtype != RF_BF16 && dtype != RF_F16) return fail(RF_ERR_ARG, "dtype must be RF_BF16 (0) or RF_F16 (1)");
  if (precision != RF_PREC_NATIVE && precision != RF_PREC_FP8)
    return fail(RF_ERR_ARG, "precision must be RF_PREC_NATIVE (0) or RF_PREC_FP8 (1)");
  return RF_OK;
}

rf_status_t check_ws(void* ws, size_t ws_bytes, const rf_ws_layout_t& lay) {
  if (!ws) return fail(RF_ERR_WORKSPACE, "workspace is NULL");
  if (reinterpret_cast<uintptr_t>(ws) & 255) return fail(RF_ERR_WORKSPACE, "workspace must be 256-byte aligned");
  if (ws_bytes < lay.total)
    return fail(RF_ERR_WORKSPACE, "workspace has %zu bytes, needs %zu", ws_bytes, lay.total);
  return RF_OK;
}

template <typename T>
T* at(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<char*>(ws) + off);
}

float resolve_scale(float scale, int D) { return (scale > 0.f && std::isfinite(scale)) ? scale : 1.0f / std::sqrt((float)D); }

// Library-owned workspace, one per device, grown on demand.
struct WsCache {
  std::mutex mu;
  void* ptr[64] = {};
  size_t bytes[64] = {};
};
WsCache g_ws, g_io;

rf_status_t cached_buffer(WsCache& c, size_t need, void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= 64) return fail(RF_ERR_UNSUPPORTED, "device index %d", dev);
  std::lock_guard<std::mutex> lock(c.mu);
  if (c.bytes[dev] < need) {
    if (c.ptr[dev]) {
      e = cudaFree(c.ptr[dev]);
      if (e != cudaSuccess) return cuda_fail(e, "cudaFree (workspace growth)");
      c.ptr[dev] = nullptr;
      c.bytes[dev] = 0;
    }
    e = cudaMalloc(&c.ptr[dev], need);
    if (e != cudaSuccess) {
      c.ptr[dev] = nullptr;
      return cuda_fail(e, "cudaMalloc (workspace)");
    }
    c.bytes[dev] = need;
  }
  *out = c.ptr[dev];
  return RF_OK;
}

// Streams and events of rf_sparse_attention_host, one set per device,
// created on first use (non-blocking streams, so a caller on the legacy
// default stream still overlaps with them): one stream for the copies in,
// one for the copies out, and one compute stream per device slot, so that
// a chunk's kernels can fill the SMs that the previous chunk's last units
// (or its second pass) leave idle.
struct HostPipe {
  cudaStream_t in = nullptr, out = nullptr, comp_s[2] = {};
  cudaEvent_t loaded[2] = {}, comp[2] = {}, stored[2] = {}, entry = nullptr;
};
std::mutex g_pipe_mu;
HostPipe g_pipe[64];
bool g_pipe_ready[64] = {};

rf_status_t host_pipe(HostPipe** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= 64) return fail(RF_ERR_UNSUPPORTED, "device index %d", dev);
  std::lock_guard<std::mutex> lock(g_pipe_mu);
  HostPipe& p = g_pipe[dev];
  if (!g_pipe_ready[dev]) {
    e = cudaStreamCreateWithFlags(&p.in, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&p.out, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&p.entry, cudaEventDisableTiming);
    for (int z = 0; z < 2 && e == cudaSuccess; ++z) {
      e = cudaStreamCreateWithFlags(&p.comp_s[z], cudaStreamNonBlocking);
      if (e != cudaSuccess) break;
      e = cudaEventCreateWithFlags(&p.loaded[z], cudaEventDisableTiming);
      if (e == cudaSuccess) e = cudaEventCreateWithFlags(&p.comp[z], cudaEventDisableTiming);
      if (e == cudaSuccess) e = cudaEventCreateWithFlags(&p.stored[z], cudaEventDisableTiming);
    }
    if (e != cudaSuccess) return cuda_fail(e, "creating the host-buffer pipeline's streams and events");
    g_pipe_ready[dev] = true;
  }
  *out = &p;
  return RF_OK;
}

}  // namespace

extern "C" {

rf_status_t rf_plan(int S, int txt_len, int T, int H, int W, int block_size, float sparsity, rf_plan_t* g) {
  if (!g) return fail(RF_ERR_ARG, "plan pointer is NULL");
  if (block_size != RF_BLOCK) return fail(RF_ERR_UNSUPPORTED, "block_size must be 128 (got %d)", block_size);
  if (!(sparsity >= 0.f && sparsity <= 1.f)) return fail(RF_ERR_ARG, "sparsity must be finite and in [0, 1]");
  if (S <= 0 || txt_len < 0 || T < 0 || H < 0 || W < 0) return fail(RF_ERR_ARG, "negative or empty size");
  if (txt_len > S) return fail(RF_ERR_ARG, "txt_len %d exceeds S %d", txt_len, S);
  const int64_t video = (int64_t)T * H * W;
  if (video != 0 && (int64_t)S != txt_len + video)
    return fail(RF_ERR_ARG, "S (%d) must equal txt_len + t*h*w (%lld)", S, (long long)(txt_len + video));
  rf_plan_t p{};
  p.S = S;
  p.txt_len = txt_len;
  p.T = T;
  p.H = H;
  p.W = W;
  p.Ha = 8 * (H / 8);
  p.Wa = 8 * (W / 8);
  int nb = 0;
  if (video != 0) {
    const int64_t aligned = (int64_t)T * p.Ha * p.Wa;
    nb = (int)(aligned / RF_BLOCK);
    p.n_tail = (int)(aligned - (int64_t)nb * RF_BLOCK);
    p.n_promoted = (int)(video - aligned);
  }
  if (video == 0 || nb < 32) {
    p.dense = 1;
    p.P = S;
    p.nb = 0;
  } else {
    if (nb > RF_MAX_BLOCKS) return fail(RF_ERR_UNSUPPORTED, "%d sparse blocks exceed the limit %d", nb, RF_MAX_BLOCKS);
    p.dense = 0;
    p.nb = nb;
    p.P = txt_len + p.n_promoted + p.n_tail;
    p.ff = std::min(nb, (p.Ha * p.Wa + RF_BLOCK - 1) / RF_BLOCK);
    const int drop = (int)std::floor((double)sparsity * nb + 1e-6);
    p.k = std::max(0, std::min(nb, nb - drop));
  }
  p.P_pad = (p.P + RF_BLOCK - 1) / RF_BLOCK * RF_BLOCK;
  if ((int64_t)p.P_pad + (int64_t)RF_BLOCK * p.nb > (int64_t)0x7FFFFF00)
    return fail(RF_ERR_UNSUPPORTED, "sequence too long");
  p.S_int = p.P_pad + RF_BLOCK * p.nb;
  p.n_tiles = p.S_int / RF_BLOCK;
  p.mask_words = (p.nb + 31) / 32;
  *g = p;
  return ok();
}

}  // extern "C"

namespace {

// The dense form of a plan: the whole sequence is the prefix, in its own order.
void densify(rf_plan_t* p) {
  p->dense = 1;
  p->P = p->S;
  p->nb = p->ff = p->k = 0;
  p->n_promoted = p->n_tail = 0;
  p->P_pad = (p->P + RF_BLOCK - 1) / RF_BLOCK * RF_BLOCK;
  p->S_int = p->P_pad;
  p->n_tiles = p->S_int / RF_BLOCK;
  p->mask_words = 0;
}

// Plans of the query geometry and of the key/value geometry (S_kv <= 0: the
// query's).  Both share txt_len; if either is dense the call is (both plans
// dense).
rf_status_t make_plans(int S, int txt_len, int T, int H, int W, int S_kv, int kv_t, int kv_h, int kv_w, int block_size,
                       float sparsity, rf_plan_t* g, rf_plan_t* gk) {
  rf_status_t st = rf_plan(S, txt_len, T, H, W, block_size, sparsity, g);
  if (st != RF_OK) return st;
  if (S_kv <= 0) {
    *gk = *g;
    return RF_OK;
  }
  if ((st = rf_plan(S_kv, txt_len, kv_t, kv_h, kv_w, block_size, sparsity, gk)) != RF_OK) return st;
  if (g->dense || gk->dense) {
    densify(g);
    densify(gk);
  }
  return RF_OK;
}

}  // namespace

extern "C" {

rf_status_t rf_plan_kv(int S, int txt_len, int T, int H, int W, int S_kv, int kv_t, int kv_h, int kv_w, int block_size,
                       float sparsity, rf_plan_t* plan, rf_plan_t* plan_kv) {
  if (!plan || !plan_kv) return fail(RF_ERR_ARG, "plan pointer is NULL");
  rf_status_t st = make_plans(S, txt_len, T, H, W, S_kv, kv_t, kv_h, kv_w, block_size, sparsity, plan, plan_kv);
  return st == RF_OK ? ok() : st;
}

rf_status_t rf_workspace_layout_ex(rf_precision_t precision, int B, int N, int D, const rf_plan_t* g,
                                   const rf_plan_t* gk, rf_ws_layout_t* lay) {
  if (!g || !lay) return fail(RF_ERR_ARG, "NULL plan or layout");
  if (!gk) gk = g;
  if (precision != RF_PREC_NATIVE && precision != RF_PREC_FP8) return fail(RF_ERR_ARG, "unknown precision %d", (int)precision);
  if (B <= 0 || N <= 0) return fail(RF_ERR_ARG, "B and N must be positive");
  if (D != RF_HEAD_DIM) return fail(RF_ERR_UNSUPPORTED, "head dim must be 128 (got %d)", D);
  const size_t heads = (size_t)B * N;
  const size_t rows_q = heads * g->S_int, rows_k = heads * gk->S_int;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at_off = off;
    off = align256(off + bytes);
    return at_off;
  };
  rf_ws_layout_t L{};
  // the work counter and the status word first: their places depend on nothing
  L.counter = take(4);
  L.status = take(4);
  // the 16-bit internal copies: native precision only (fp8 stage 1 writes e4m3 codes instead)
  const bool fp8 = precision == RF_PREC_FP8;
  L.q_int = take(fp8 ? 0 : rows_q * RF_HEAD_DIM * 2);
  L.k_int = take(fp8 ? 0 : rows_k * RF_HEAD_DIM * 2);
  L.v_int = take(fp8 ? 0 : rows_k * RF_HEAD_DIM * 2);
  L.pooled_q = take(heads * g->nb * RF_HEAD_DIM * 4);
  L.pooled_k = take(heads * gk->nb * RF_HEAD_DIM * 4);
  L.mask = take(heads * g->nb * gk->mask_words * 4);
  L.kept = take(heads * g->nb * 4);
  L.margin = take(heads * g->nb * 4);
  L.q8 = take(fp8 ? rows_q * RF_HEAD_DIM : 0);
  L.k8 = take(fp8 ? rows_k * RF_HEAD_DIM : 0);
  L.v8 = take(fp8 ? rows_k * RF_HEAD_DIM : 0);
  L.scales = take(fp8 ? heads * (g->n_tiles + 2 * (size_t)gk->n_tiles) * 4 : 0);
  L.vmax = take(fp8 ? heads * 4 : 0);
  L.redo = take((2 + heads * g->n_tiles) * 4);
  L.total = off;
  *lay = L;
  return ok();
}

rf_status_t rf_workspace_layout(int B, int N, int D, const rf_plan_t* g, rf_ws_layout_t* lay) {
  return rf_workspace_layout_ex(RF_PREC_NATIVE, B, N, D, g, nullptr, lay);
}

size_t rf_workspace_size_ex(rf_precision_t precision, int B, int S, int N, int D, int txt_len, int T, int H, int W,
                            int S_kv, int kv_t, int kv_h, int kv_w) {
  rf_plan_t g, gk;
  rf_ws_layout_t L;
  if (make_plans(S, txt_len, T, H, W, S_kv, kv_t, kv_h, kv_w, RF_BLOCK, 0.f, &g, &gk) != RF_OK) return 0;
  if (rf_workspace_layout_ex(precision, B, N, D, &g, &gk, &L) != RF_OK) return 0;
  return L.total;
}

size_t rf_workspace_size(int B, int S, int N, int D, int txt_len, int T, int H, int W) {
  return rf_workspace_size_ex(RF_PREC_NATIVE, B, S, N, D, txt_len, T, H, W, 0, 0, 0, 0);
}

rf_status_t rf_prepare_ex(const void* q, const void* k, const void* v, rf_dtype_t dtype, rf_precision_t precision,
                          rf_layout_t layout, int B, int S, int N, int D, int txt_len, int T, int H, int W, int S_kv,
                          int kv_t, int kv_h, int kv_w, int block_size, float sparsity, void* ws, size_t ws_bytes,
                          void* stream) {
  rf_status_t st = check_common(layout, B, S, N, D);
  if (st != RF_OK) return st;
  if ((st = check_types(dtype, precision)) != RF_OK) return st;
  if (!q || !k || !v) return fail(RF_ERR_ARG, "q, k and v must be device pointers");
  if ((st = check_aligned16(q, "q")) != RF_OK || (st = check_aligned16(k, "k")) != RF_OK ||
      (st = check_aligned16(v, "v")) != RF_OK)
    return st;
  rf_plan_t g, gk;
  if ((st = make_plans(S, txt_len, T, H, W, S_kv, kv_t, kv_h, kv_w, block_size, sparsity, &g, &gk)) != RF_OK)
    return st;
  rf_ws_layout_t L;
  if ((st = rf_workspace_layout_ex(precision, B, N, D, &g, &gk, &L)) != RF_OK) return st;
  if ((st = check_ws(ws, ws_bytes, L)) != RF_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  NvtxRange range("rf prepare: K1 reorder + block means, K2 scores + top-k");
  cudaError_t e =
      precision == RF_PREC_FP8
          ? rf::launch_permute_pool_fp8(q, k, v, dtype, layout, B, S, gk.S, N, g, gk, at<uint8_t>(ws, L.q8),
                                        at<uint8_t>(ws, L.k8), at<uint8_t>(ws, L.v8), at<float>(ws, L.scales),
                                        at<float>(ws, L.vmax), at<float>(ws, L.pooled_q), at<float>(ws, L.pooled_k), s)
          : rf::launch_permute_pool(q, k, v, dtype, layout, B, S, gk.S, N, g, gk, at<void>(ws, L.q_int),
                                    at<void>(ws, L.k_int), at<void>(ws, L.v_int), at<float>(ws, L.pooled_q),
                                    at<float>(ws, L.pooled_k), s);
  if (e != cudaSuccess) return cuda_fail(e, "permute/pool launch");
  cudaEvent_t stage_event;
  {
    std::lock_guard<std::mutex> lock(g_debug_mu);
    stage_event = g_stage_event;
  }
  if (stage_event && (e = cudaEventRecord(stage_event, s)) != cudaSuccess) return cuda_fail(e, "stage event record");
  e = rf::launch_mask(at<float>(ws, L.pooled_q), at<float>(ws, L.pooled_k), B * N, g, gk, at<uint32_t>(ws, L.mask),
                      at<int>(ws, L.kept), at<float>(ws, L.margin), s);
  if (e != cudaSuccess) return cuda_fail(e, "mask launch");
  return ok();
}

rf_status_t rf_prepare(const void* q, const void* k, const void* v, rf_layout_t layout, int B, int S, int N, int D,
                       int txt_len, int T, int H, int W, int block_size, float sparsity, void* ws, size_t ws_bytes,
                       void* stream) {
  return rf_prepare_ex(q, k, v, RF_BF16, RF_PREC_NATIVE, layout, B, S, N, D, txt_len, T, H, W, 0, 0, 0, 0, block_size,
                       sparsity, ws, ws_bytes, stream);
}

rf_status_t rf_attend_ex(rf_dtype_t dtype, rf_precision_t precision, rf_layout_t layout, int B, int S, int N, int D,
                         int txt_len, int T, int H, int W, int S_kv, int kv_t, int kv_h, int kv_w, int block_size,
                         float sparsity, float scale, void* out, void* ws, size_t ws_bytes, void* stream) {
  rf_status_t st = check_common(layout, B, S, N, D);
  if (st != RF_OK) return st;
  if ((st = check_types(dtype, precision)) != RF_OK) return st;
  if (!out) return fail(RF_ERR_ARG, "out must be a device pointer");
  if ((st = check_aligned16(out, "out")) != RF_OK) return st;
  rf_plan_t g, gk;
  if ((st = make_plans(S, txt_len, T, H, W, S_kv, kv_t, kv_h, kv_w, block_size, sparsity, &g, &gk)) != RF_OK)
    return st;
  rf_ws_layout_t L;
  if ((st = rf_workspace_layout_ex(precision, B, N, D, &g, &gk, &L)) != RF_OK) return st;
  if ((st = check_ws(ws, ws_bytes, L)) != RF_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  NvtxRange range("rf attend: K3 block-sparse attention");
  cudaError_t e = cudaMemsetAsync(at<int>(ws, L.status), 0, sizeof(int), s);
  if (e != cudaSuccess) return cuda_fail(e, "clearing the status word");
  if (precision == RF_PREC_FP8)
    e = rf::launch_attention_fp8(at<uint8_t>(ws, L.q8), at<uint8_t>(ws, L.k8), at<uint8_t>(ws, L.v8),
                                 at<float>(ws, L.scales), at<float>(ws, L.vmax), at<uint32_t>(ws, L.mask), dtype,
                                 layout, B, S, N, g, gk, resolve_scale(scale, D), out, at<int>(ws, L.counter),
                                 at<int>(ws, L.status), at<int>(ws, L.redo), debug_settings(), s);
  else
    e = rf::launch_attention(at<void>(ws, L.q_int), at<void>(ws, L.k_int), at<void>(ws, L.v_int),
                             at<uint32_t>(ws, L.mask), dtype, layout, B, S, N, g, gk, resolve_scale(scale, D), out,
                             at<int>(ws, L.counter), at<int>(ws, L.status), at<int>(ws, L.redo), debug_settings(), s);
  if (e != cudaSuccess) return cuda_fail(e, "attention launch");
  return ok();
}

rf_status_t rf_attend(rf_layout_t layout, int B, int S, int N, int D, int txt_len, int T, int H, int W,
                      int block_size, float sparsity, float scale, void* out, void* ws, size_t ws_bytes,
                      void* stream) {
  return rf_attend_ex(RF_BF16, RF_PREC_NATIVE, layout, B, S, N, D, txt_len, T, H, W, 0, 0, 0, 0, block_size, sparsity,
                      scale, out, ws, ws_bytes, stream);
}

rf_status_t rf_sparse_attention_ex(const void* q, const void* k, const void* v, rf_dtype_t dtype,
                                   rf_precision_t precision, rf_layout_t layout, int B, int S, int N, int D,
                                   int txt_len, int T, int H, int W, int S_kv, int kv_t, int kv_h, int kv_w,
                                   int block_size, float sparsity, float scale, void* out, void* ws, size_t ws_bytes,
                                   void* stream) {
  rf_status_t st = check_common(layout, B, S, N, D);
  if (st != RF_OK) return st;
  if ((st = check_types(dtype, precision)) != RF_OK) return st;
  if (!q || !k || !v || !out) return fail(RF_ERR_ARG, "q, k, v and out must be device pointers");
  if (out == q || out == k || out == v) return fail(RF_ERR_ARG, "out must not alias q, k or v");
  if ((st = check_aligned16(q, "q")) != RF_OK || (st = check_aligned16(k, "k")) != RF_OK ||
      (st = check_aligned16(v, "v")) != RF_OK || (st = check_aligned16(out, "out")) != RF_OK)
    return st;
  if (!ws) {
    rf_plan_t g, gk;
    if ((st = make_plans(S, txt_len, T, H, W, S_kv, kv_t, kv_h, kv_w, block_size, sparsity, &g, &gk)) != RF_OK)
      return st;
    rf_ws_layout_t L;
    if ((st = rf_workspace_layout_ex(precision, B, N, D, &g, &gk, &L)) != RF_OK) return st;
    if ((st = cached_buffer(g_ws, L.total, &ws)) != RF_OK) return st;
    ws_bytes = L.total;
  }
  st = rf_prepare_ex(q, k, v, dtype, precision, layout, B, S, N, D, txt_len, T, H, W, S_kv, kv_t, kv_h, kv_w,
                     block_size, sparsity, ws, ws_bytes, stream);
  if (st != RF_OK) return st;
  return rf_attend_ex(dtype, precision, layout, B, S, N, D, txt_len, T, H, W, S_kv, kv_t, kv_h, kv_w, block_size,
                      sparsity, scale, out, ws, ws_bytes, stream);
}

rf_status_t rf_sparse_attention_ws(const void* q, const void* k, const void* v, rf_layout_t layout, int B, int S,
                                   int N, int D, int txt_len, int T, int H, int W, int block_size, float sparsity,
                                   float scale, void* out, void* ws, size_t ws_bytes, void* stream) {
  if (!ws) return fail(RF_ERR_WORKSPACE, "workspace is NULL");
  return rf_sparse_attention_ex(q, k, v, RF_BF16, RF_PREC_NATIVE, layout, B, S, N, D, txt_len, T, H, W, 0, 0, 0, 0,
                                block_size, sparsity, scale, out, ws, ws_bytes, stream);
}

rf_status_t rf_sparse_attention(const void* q, const void* k, const void* v, rf_layout_t layout, int B, int S, int N,
                                int D, int txt_len, int T, int H, int W, int block_size, float sparsity, float scale,
                                void* out, void* stream) {
  return rf_sparse_attention_ex(q, k, v, RF_BF16, RF_PREC_NATIVE, layout, B, S, N, D, txt_len, T, H, W, 0, 0, 0, 0,
                                block_size, sparsity, scale, out, nullptr, 0, stream);
}

rf_status_t rf_unpermute(const void* o_int, rf_layout_t layout, int B, int S, int N, int D, int txt_len, int T, int H,
                         int W, void* out, void* stream) {
  rf_status_t st = check_common(layout, B, S, N, D);
  if (st != RF_OK) return st;
  if (!o_int || !out) return fail(RF_ERR_ARG, "o_int and out must be device pointers");
  if ((st = check_aligned16(o_int, "o_int")) != RF_OK || (st = check_aligned16(out, "out")) != RF_OK) return st;
  rf_plan_t g;
  if ((st = rf_plan(S, txt_len, T, H, W, RF_BLOCK, 0.f, &g)) != RF_OK) return st;
  cudaError_t e = rf::launch_unpermute(o_int, layout, B, S, N, g, out, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "unpermute launch");
  return ok();
}

rf_status_t rf_sparse_attention_host_ex(const void* qh, const void* kh, const void* vh, rf_dtype_t dtype,
                                        rf_precision_t precision, rf_layout_t layout, int B, int S, int N, int D,
                                        int txt_len, int T, int H, int W, int S_kv, int kv_t, int kv_h, int kv_w,
                                        int block_size, float sparsity, float scale, void* out_h, void* stream) {
  rf_status_t st = check_common(layout, B, S, N, D);
  if (st != RF_OK) return st;
  if ((st = check_types(dtype, precision)) != RF_OK) return st;
  if (!qh || !kh || !vh || !out_h) return fail(RF_ERR_ARG, "host buffers must not be NULL");
  rf_plan_t g, gk;
  if ((st = make_plans(S, txt_len, T, H, W, S_kv, kv_t, kv_h, kv_w, block_size, sparsity, &g, &gk)) != RF_OK)
    return st;
  // Heads are independent in every precision (the fp8 scales belong to one
  // head's tiles, vmax to one head), so the call runs on chunks of c heads
  // of one batch entry, each a [1, S, c, D] (BSND) or [1, c, S, D] (BNSD)
  // problem, in two device slots.  While chunk i computes on its slot's
  // stream (after the work already queued on the caller's stream), chunk
  // i + 1 is copied in on one stream and chunk i - 1 copied out on another;
  // chunk i + 1 may start computing before chunk i's last units are done.  About 96 MiB of q, k and v per chunk (2 heads at
  // MiniMax-H3): a shorter pipeline tail than 192 MiB (52.3 vs 53.4 ms per
  // call there).  At least 2 heads when BSND: a chunk of 1 head copies
  // 256-byte rows, and the strided copy then runs far below the link's rate
  // (81.6 ms).
  const int S_k = S_kv > 0 ? S_kv : S;
  const size_t head_q = (size_t)S * D * 2, head_k = (size_t)S_k * D * 2;
  int c = std::max(1, std::min(N, (int)(((size_t)96 << 20) / (head_q + 2 * head_k))));
  if (layout == RF_BSND && c < 2) c = std::min(N, 2);
  const size_t chunk_q = align256((size_t)c * head_q), chunk_k = align256((size_t)c * head_k);
  const size_t slot = 2 * chunk_q + 2 * chunk_k;   // q, k, v, out
  rf_ws_layout_t L;
  if ((st = rf_workspace_layout_ex(precision, 1, c, D, &g, &gk, &L)) != RF_OK) return st;
  const size_t ws_slot = align256(L.total);
  void* io = nullptr;
  void* ws = nullptr;
  if ((st = cached_buffer(g_io, 2 * slot, &io)) != RF_OK) return st;
  if ((st = cached_buffer(g_ws, 2 * ws_slot, &ws)) != RF_OK) return st;
  HostPipe* hp = nullptr;
  if ((st = host_pipe(&hp)) != RF_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  {
    cudaError_t e0 = cudaEventRecord(hp->entry, s);
    for (int z = 0; z < 2 && e0 == cudaSuccess; ++z) e0 = cudaStreamWaitEvent(hp->comp_s[z], hp->entry, 0);
    if (e0 != cudaSuccess) return cuda_fail(e0, "ordering the host-buffer pipeline after the caller's stream");
  }
  // every stream the call used has drained (also on an error: no copy of the
  // caller's buffers may still run when this returns)
  auto drain = [&]() {
    cudaError_t r = cudaSuccess;
    for (cudaStream_t x : {hp->in, hp->out, hp->comp_s[0], hp->comp_s[1], s}) {
      const cudaError_t ex = cudaStreamSynchronize(x);
      if (r == cudaSuccess) r = ex;
    }
    return r;
  };
  const bool bsnd = layout == RF_BSND;
  const size_t row = (size_t)N * D * 2;   // BSND: one token's heads
  // `heads` heads of a tensor of `len` tokens; BSND copies `len` strided rows
  auto copy = [&](void* dst, const void* src, int heads, int len, cudaMemcpyKind kind, bool to_dev, cudaStream_t cs) {
    if (!bsnd) return cudaMemcpyAsync(dst, src, (size_t)heads * len * D * 2, kind, cs);
    const size_t w = (size_t)heads * D * 2;
    return to_dev ? cudaMemcpy2DAsync(dst, w, src, row, w, len, kind, cs)
                  : cudaMemcpy2DAsync(dst, row, src, w, w, len, kind, cs);
  };
  const char* srcs[3] = {static_cast<const char*>(qh), static_cast<const char*>(kh), static_cast<const char*>(vh)};
  char* outh = static_cast<char*>(out_h);
  int i = 0;
  cudaError_t e = cudaSuccess;
  for (int b = 0; b < B; ++b) {
    for (int n0 = 0; n0 < N; n0 += c, ++i) {
      const int heads = std::min(c, N - n0);
      const int z = i & 1;
      char* d = static_cast<char*>(io) + (size_t)z * slot;
      char* dev[4] = {d, d + chunk_q, d + chunk_q + chunk_k, d + chunk_q + 2 * chunk_k};   // q, k, v, out
      // host offset of the chunk's first element in a tensor of `len` tokens
      auto off = [&](int len) {
        return bsnd ? ((size_t)b * len * N + n0) * D * 2 : ((size_t)b * N + n0) * len * D * 2;
      };
      // copy in once the slot's previous chunk has been computed
      if (i >= 2 && (e = cudaStreamWaitEvent(hp->in, hp->comp[z], 0)) != cudaSuccess) break;
      for (int t = 0; t < 3 && e == cudaSuccess; ++t) {
        const int len = t == 0 ? S : S_k;
        e = copy(dev[t], srcs[t] + off(len), heads, len, cudaMemcpyHostToDevice, true, hp->in);
      }
      if (e != cudaSuccess || (e = cudaEventRecord(hp->loaded[z], hp->in)) != cudaSuccess) break;
      // compute once it is in and the slot's previous output has left
      cudaStream_t cs = hp->comp_s[z];
      if ((e = cudaStreamWaitEvent(cs, hp->loaded[z], 0)) != cudaSuccess) break;
      if (i >= 2 && (e = cudaStreamWaitEvent(cs, hp->stored[z], 0)) != cudaSuccess) break;
      st = rf_sparse_attention_ex(dev[0], dev[1], dev[2], dtype, precision, layout, 1, S, heads, D, txt_len, T, H,
                                  W, S_kv, kv_t, kv_h, kv_w, block_size, sparsity, scale, dev[3],
                                  static_cast<char*>(ws) + (size_t)z * ws_slot, ws_slot, cs);
      if (st != RF_OK) {
        drain();
        return st;
      }
      if ((e = cudaEventRecord(hp->comp[z], cs)) != cudaSuccess) break;
      // copy out
      if ((e = cudaStreamWaitEvent(hp->out, hp->comp[z], 0)) != cudaSuccess) break;
      if ((e = copy(outh + off(S), dev[3], heads, S, cudaMemcpyDeviceToHost, false, hp->out)) != cudaSuccess) break;
      if ((e = cudaEventRecord(hp->stored[z], hp->out)) != cudaSuccess) break;
    }
    if (e != cudaSuccess) break;
  }
  const cudaError_t e_drain = drain();
  if (e == cudaSuccess) e = e_drain;
  if (e != cudaSuccess) return cuda_fail(e, "host-buffer pipeline (copies, events or synchronisation)");
  return ok();
}

rf_status_t rf_sparse_attention_host(const void* qh, const void* kh, const void* vh, rf_layout_t layout, int B, int S,
                                     int N, int D, int txt_len, int T, int H, int W, int block_size, float sparsity,
                                     float scale, void* out_h, void* stream) {
  return rf_sparse_attention_host_ex(qh, kh, vh, RF_BF16, RF_PREC_NATIVE, layout, B, S, N, D, txt_len, T, H, W, 0, 0,
                                     0, 0, block_size, sparsity, scale, out_h, stream);
}

rf_status_t rf_read_status(void* ws, size_t ws_bytes, int B, int N, int D, const rf_plan_t* g, int* status,
                           void* stream) {
  if (!status) return fail(RF_ERR_ARG, "status pointer is NULL");
  rf_ws_layout_t L;
  rf_status_t st = rf_workspace_layout(B, N, D, g, &L);   // validates the arguments; the status word's place
  if (st != RF_OK) return st;                             // does not depend on them
  if (!ws) return fail(RF_ERR_WORKSPACE, "workspace is NULL");
  if (reinterpret_cast<uintptr_t>(ws) & 255) return fail(RF_ERR_WORKSPACE, "workspace must be 256-byte aligned");
  if (ws_bytes < L.status + sizeof(int)) return fail(RF_ERR_WORKSPACE, "workspace too small for its status word");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int h = 0;
  cudaError_t e = cudaMemcpyAsync(&h, at<int>(ws, L.status), sizeof(int), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaMemsetAsync(at<int>(ws, L.status), 0, sizeof(int), s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "reading the status word");
  *status = h;
  return ok();
}

rf_status_t rf_read_stats_ex(rf_precision_t precision, void* ws, size_t ws_bytes, int B, int N, int D,
                             const rf_plan_t* g, const rf_plan_t* gk, rf_stats_t* stats, void* stream) {
  if (!stats) return fail(RF_ERR_ARG, "stats pointer is NULL");
  if (!g) return fail(RF_ERR_ARG, "plan pointer is NULL");
  if (!gk) gk = g;
  rf_ws_layout_t L;
  rf_status_t st = rf_workspace_layout_ex(precision, B, N, D, g, gk, &L);
  if (st != RF_OK) return st;
  if ((st = check_ws(ws, ws_bytes, L)) != RF_OK) return st;
  const size_t heads = (size_t)B * N, rows = heads * g->nb;
  std::vector<int> kept(rows);
  std::vector<float> margin(rows);
  int redo[2] = {0, 0}, status = 0;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaSuccess;
  if (rows) {
    e = cudaMemcpyAsync(kept.data(), at<int>(ws, L.kept), rows * sizeof(int), cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(margin.data(), at<float>(ws, L.margin), rows * sizeof(float), cudaMemcpyDeviceToHost, s);
  }
  if (e == cudaSuccess) e = cudaMemcpyAsync(redo, at<int>(ws, L.redo), sizeof(redo), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaMemcpyAsync(&status, at<int>(ws, L.status), sizeof(int), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "reading the workspace statistics");
  rf_stats_t r{};
  const double S = g->S, S_kv = gk->S;
  if (g->dense) {
    r.kept_pairs = (double)heads * S * S_kv;
  } else {
    // dense query rows (prefix, first-frame blocks) read every key; a sparse
    // block's rows read the key prefix and 128 keys per kept key block
    const double dense_rows = (double)g->P + 128.0 * g->ff;
    double sparse_keys = 0;
    for (size_t h = 0; h < heads; ++h)
      for (int i = g->ff; i < g->nb; ++i) {
        const size_t j = h * g->nb + i;
        r.kept_blocks += kept[j];
        sparse_keys += 128.0 * kept[j] + gk->P;
        if (margin[j] < 1e-5f) ++r.near_ties;
      }
    r.query_blocks = (long long)heads * (g->nb - g->ff);
    r.kept_pairs = (double)heads * dense_rows * S_kv + 128.0 * sparse_keys;
  }
  r.density = r.kept_pairs / ((double)heads * S * S_kv);
  r.redo_tiles = redo[1] < 0 ? (int)(heads * g->n_tiles) : redo[1];
  r.status = status;
  *stats = r;
  return ok();
}

rf_status_t rf_read_stats(void* ws, size_t ws_bytes, int B, int N, int D, const rf_plan_t* g, rf_stats_t* stats,
                          void* stream) {
  return rf_read_stats_ex(RF_PREC_NATIVE, ws, ws_bytes, B, N, D, g, nullptr, stats, stream);
}

rf_status_t rf_block_mask_noalloc(const void* q, const void* k, rf_layout_t layout, int B, int S, int N, int D,
                                  int txt_len, int T, int H, int W, int block_size, float sparsity, uint32_t* mask,
                                  int32_t* kept, float* margin, void* stream) {
  rf_status_t st = check_common(layout, B, S, N, D);
  if (st != RF_OK) return st;
  if (!q || !k) return fail(RF_ERR_ARG, "q and k must be device pointers");
  if ((st = check_aligned16(q, "q")) != RF_OK || (st = check_aligned16(k, "k")) != RF_OK) return st;
  rf_plan_t g;
  if ((st = rf_plan(S, txt_len, T, H, W, block_size, sparsity, &g)) != RF_OK) return st;
  if (g.nb == 0) return ok();
  if (!mask || !kept || !margin) return fail(RF_ERR_ARG, "mask, kept and margin must be device pointers");
  if ((reinterpret_cast<uintptr_t>(mask) | reinterpret_cast<uintptr_t>(kept) | reinterpret_cast<uintptr_t>(margin)) & 3)
    return fail(RF_ERR_ARG, "mask, kept and margin must be 4-byte aligned");
  const size_t need = (size_t)B * N * g.nb * RF_HEAD_DIM * sizeof(float) * 2;
  if (need > RF_NOALLOC_SCRATCH_BYTES)
    return fail(RF_ERR_UNSUPPORTED,
                "B*N*nb = %zu block rows need %zu bytes of pooled scratch, above the static %u-byte array",
                (size_t)B * N * g.nb, need, (unsigned)RF_NOALLOC_SCRATCH_BYTES);
  cudaError_t e = rf::launch_block_mask_noalloc(q, k, RF_BF16, layout, B, S, N, g, mask, kept, margin,
                                                static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "no-allocation mask launch");
  return ok();
}

rf_status_t rf_debug_set_wait(long long wait_limit_ns, int skip_first_q) {
  if (wait_limit_ns < 0 || (skip_first_q != 0 && skip_first_q != 1))
    return fail(RF_ERR_ARG, "wait limit must be >= 0 and skip_first_q 0 or 1");
  std::lock_guard<std::mutex> lock(g_debug_mu);
  g_debug.wait_limit_ns = wait_limit_ns;
  g_debug.skip_first_q = skip_first_q;
  return ok();
}

rf_status_t rf_debug_set_path(int path, float sum_limit) {
  if ((path != 0 && path != 1) || !(sum_limit >= 0.f))
    return fail(RF_ERR_ARG, "path must be 0 or 1 and sum_limit >= 0");
  std::lock_guard<std::mutex> lock(g_debug_mu);
  g_debug.path = path;
  g_debug.sum_limit = sum_limit;
  return ok();
}

rf_status_t rf_debug_set_stage_event(void* event) {
  std::lock_guard<std::mutex> lock(g_debug_mu);
  g_stage_event = static_cast<cudaEvent_t>(event);
  return ok();
}

rf_status_t rf_debug_exp2_poly(const float* x, float* y, int n, void* stream) {
  if (n < 0) return fail(RF_ERR_ARG, "n must be >= 0");
  if (n > 0 && (!x || !y)) return fail(RF_ERR_ARG, "x and y must be device pointers");
  if ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(y)) & 3)
    return fail(RF_ERR_ARG, "x and y must be 4-byte aligned");
  cudaError_t e = rf::launch_debug_exp2_poly(x, y, n, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "exp2 polynomial launch");
  return ok();
}

const char* rf_last_error_string(void) { return g_last_error.c_str(); }

}  // extern "C"
