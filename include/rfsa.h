/*
 * rfsa.h -- C ABI of the RainFusion rf_v2 block-sparse video attention
 * library for NVIDIA B200 (sm_100a).
 *
 * The operation is the rf_v2 mode of MindSpore Lite's
 * "lite_boost.ops.sparse_attention" (pipeline: token reorder -> block
 * pooling -> top-k sparse mask -> rain_fusion_attention -> inverse reorder),
 * with the geometry and dense-fallback rules of the vllm-omni user guide
 * page "RainFusion Attention" (intro; "Configuration"; "Geometry handling").
 *
 * Each declaration below names the passage that defines it: [SA] is
 * MindSpore Lite "lite_boost.ops.sparse_attention" (its pipeline line, its
 * parameter list, "Returns" and "Raises"); [RF] is the vllm-omni user guide
 * page "RainFusion Attention" (intro, "Configuration", "Requirements and
 * compatibility", "Geometry handling").  Entry points marked "library"
 * have no counterpart on the pages: they expose the stages, buffers and
 * test controls of this implementation.
 *
 * Conventions for every entry point:
 *  - q, k, v, out: DEVICE pointers to bf16 (fp16 through the _ex entry
 *    points with dtype RF_F16), caller-owned, contiguous, 16-byte aligned
 *    (the kernels move 16-byte vectors; a misaligned pointer is RF_ERR_ARG),
 *    in the layout given (RF_BSND = [B, S, N, D], RF_BNSD = [B, N, S, D]);
 *    out has the shape, layout and element type of q and must not alias q,
 *    k or v.
 *  - D and block_size must be 128.
 *  - S = txt_len + latent_t * latent_h * latent_w.  latent (0, 0, 0) means
 *    "no video geometry": the call is dense softmax attention over S.
 *  - sparsity must be finite and in [0, 1]; it is the nominal fraction of
 *    key blocks dropped per query block (0 = dense).
 *  - scale <= 0 or NaN selects head_dim ** -0.5.
 *  - Argument errors are returned before anything is enqueued.  Work is
 *    enqueued on `stream` (NULL = legacy default stream) and is asynchronous;
 *    launch failures return RF_ERR_CUDA.  Nothing here synchronises except
 *    rf_read_status and rf_read_stats(_ex) (the stream given) and
 *    rf_sparse_attention_host(_ex) (its streams).
 *  - A device-side wait that runs past its time limit makes the kernel
 *    record RF_ERR_TIMEOUT in the workspace status word and return early;
 *    rf_read_status reports it.
 *  - The library never frees caller memory.
 *  - On error, rf_last_error_string() (thread-local) says why.
 */
#ifndef RFSA_H
#define RFSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* [SA] parameter input_layout: "BSND" or "BNSD". */
typedef enum { RF_BSND = 0, RF_BNSD = 1 } rf_layout_t;

/* Element type of q, k, v and out.  [SA] intro: input tensors may be
 * float16 or bfloat16. */
typedef enum { RF_BF16 = 0, RF_F16 = 1 } rf_dtype_t;

/* Arithmetic of the attention's two products.  [RF] "Configuration",
 * precision "bf16" (the default) or "fp8" (the "mix" mode is not offered).
 * RF_PREC_NATIVE: Q K^T and P V
 * on the tensor cores in the input type (bf16 or fp16) with fp32
 * accumulation.  RF_PREC_FP8: Q, K and V quantised to fp8 e4m3 with one
 * fp32 scale per 128-row block of the internal layout (per tensor and head:
 * scale = amax(|x|) over the block / 448, code = e4m3 round-to-nearest-even
 * with saturation of x * (448 / amax), all-zero blocks get scale 0); Q K^T
 * and P V then run as e4m3 x e4m3 tensor-core products with fp32
 * accumulation, P quantised to e4m3 per tile.  The block mask is the same in
 * both: it is computed from the unquantised inputs. */
typedef enum { RF_PREC_NATIVE = 0, RF_PREC_FP8 = 1 } rf_precision_t;

/* Return codes.  RF_ERR_LAYOUT is [SA] "Raises" (ValueError on input_layout);
 * the sparsity range is [SA] parameter sparsity and [RF] "Configuration";
 * the others are library codes. */
typedef enum {
  RF_OK = 0,
  RF_ERR_LAYOUT = 1,      /* layout not BSND/BNSD (the page's ValueError on input_layout) */
  RF_ERR_ARG = 2,         /* bad sizes, sparsity outside [0, 1], S != txt_len + t*h*w, NULL or misaligned pointer */
  RF_ERR_UNSUPPORTED = 3, /* D != 128, block_size != 128, or more sparse blocks than RF_MAX_BLOCKS */
  RF_ERR_CUDA = 4,        /* a CUDA runtime call or launch failed */
  RF_ERR_WORKSPACE = 5,   /* workspace too small or misaligned */
  RF_ERR_TIMEOUT = 6      /* a device-side wait ran past its limit (read via rf_read_status) */
} rf_status_t;

/* [SA] parameter block_size (default 128; the only size supported here) and
 * the head dim of every workload on the pages (MiniMax-H3: 56 heads x 128). */
#define RF_HEAD_DIM 128
#define RF_BLOCK 128
/* Library limit on sparse blocks per clip (524,288 aligned video tokens). */
#define RF_MAX_BLOCKS 4096

/* Geometry of one clip, shared by every (batch, head).  [RF] "Geometry
 * handling" (8x8-aligned spatial arrangement, the promoted suffix, the
 * 62,496 / 2,976 / 465 x 128 worked example) and intro (128-token blocks,
 * (t, h, w) order, first-frame blocks dense, fewer than 32 blocks dense);
 * [SA] parameters txt_len and latent_shape_q.
 * Internal row order per (b, head): [prefix: text, promoted video tokens in
 * natural (t, h, w) order, aligned tokens past the last whole block]
 * [zero pad to a multiple of 128] [nb sparse blocks of 128 rows, each two
 * 8x8 tiles: frames in order, tiles row-major, raster inside a tile]. */
typedef struct {
  int S, txt_len, T, H, W;
  int Ha, Wa;        /* 8 * floor(H / 8), 8 * floor(W / 8) */
  int n_promoted;    /* video tokens outside the Ha x Wa grid */
  int n_tail;        /* aligned tokens past the last whole 128-block */
  int P;             /* dense prefix rows (S when dense) */
  int P_pad;         /* P rounded up to 128 */
  int nb;            /* sparse 128-blocks (0 when dense) */
  int ff;            /* first-frame blocks: ceil(Ha * Wa / 128), at most nb */
  int k;             /* top-k kept per sparse query block: nb - floor(sparsity * nb + 1e-6) */
  int dense;         /* 1: every row attends to every key (no geometry, or nb < 32) */
  int S_int;         /* internal rows per (b, head) = P_pad + 128 * nb */
  int n_tiles;       /* S_int / 128 */
  int mask_words;    /* 32-bit words per mask row = ceil(nb / 32) */
} rf_plan_t;

/* Library: byte offsets of the regions of a workspace (all 256-byte aligned).
 * q_int/k_int/v_int: 16-bit (input type) [B, N, S_int, 128], native
 * precision only (zero-sized with RF_PREC_FP8); pooled_q/pooled_k: fp32
 * [B, N, nb, 128] (block means); mask: uint32 [B, N, nb, mask_words], bit j
 * of row i set when query block i reads key block j; kept: int32 [B, N, nb]
 * (bits set per row); margin: fp32 [B, N, nb] (relative gap between the
 * k-th and (k+1)-th block score of the row, +inf when not defined);
 * counter: int32 work counter; status: int32 device status word (both at
 * the start of the workspace, whatever the geometry).
 * With a key/value geometry of its own, k_int/v_int/pooled_k and the mask
 * columns follow the key plan.
 * Only with RF_PREC_FP8 (zero-sized otherwise): q8/k8: e4m3 codes
 * [B, N, S_int, 128]; v8: e4m3 codes of V with each 128-row block stored
 * transposed ([B, N, n_tiles, 128 channels, 128 rows]); scales: fp32
 * q [B, N, n_tiles_q], then k and v [B, N, n_tiles_kv]; vmax: fp32 [B, N],
 * the largest V block scale of each head.
 * redo: int32 [2 + B * N * n_tiles_q], the query tiles the attention hands
 * to its second pass ([0] a work counter, [1] how many, [2 ...] their ids). */
typedef struct {
  size_t q_int, k_int, v_int, pooled_q, pooled_k, mask, kept, margin, counter, status;
  size_t q8, k8, v8, scales, vmax;
  size_t redo;
  size_t total;
} rf_ws_layout_t;

/* Library: statistics of the last call on a workspace (rf_read_stats).  The
 * near-tie count is the one the mask's bit-exact check excuses. */
typedef struct {
  long long kept_blocks;   /* key blocks kept over all sparse query blocks (top-k plus forced first-frame columns) */
  long long query_blocks;  /* sparse query blocks that select (B * N * (nb - ff)) */
  double kept_pairs;       /* (query row, key) pairs attended: dense rows read all S keys, a sparse block's rows
                            * the P prefix keys plus 128 per kept block; 4 * D * kept_pairs is the kept-block work */
  double density;          /* kept_pairs / (B * N * S * S) */
  int near_ties;           /* sparse query blocks whose k-th and (k+1)-th block scores are within 1e-5 (relative) */
  int redo_tiles;          /* query tiles the attention handed to its second pass (P beyond its type's headroom) */
  int status;              /* the workspace status word (not cleared) */
} rf_stats_t;

/* Host-only: validate a geometry and fill *plan.  No CUDA call.  [RF]
 * "Geometry handling" and intro; [SA] parameters txt_len, block_size,
 * latent_shape_q, sparsity (k = nb - floor(sparsity * nb + 1e-6)). */
rf_status_t rf_plan(int S, int txt_len, int latent_t, int latent_h, int latent_w, int block_size, float sparsity,
                    rf_plan_t* plan);

/* Host-only: the plans of a call whose keys and values have a geometry of
 * their own ([SA] parameter latent_shape_k, which defaults to latent_shape_q) (S_kv, kv_t, kv_h, kv_w as in rf_prepare_ex; S_kv <= 0: the
 * query's, and *plan_kv = *plan).  If either geometry is dense both plans
 * come back dense (the whole sequence as the prefix, in its own order). */
rf_status_t rf_plan_kv(int S, int txt_len, int latent_t, int latent_h, int latent_w, int S_kv, int kv_t, int kv_h,
                       int kv_w, int block_size, float sparsity, rf_plan_t* plan, rf_plan_t* plan_kv);

/* Library, host-only: workspace regions for B x N heads of head dim D under `plan`. */
rf_status_t rf_workspace_layout(int B, int N, int D, const rf_plan_t* plan, rf_ws_layout_t* layout);

/* Library, host-only: bytes of workspace rf_sparse_attention_ws needs (0 on bad arguments). */
size_t rf_workspace_size(int B, int S, int N, int D, int txt_len, int latent_t, int latent_h, int latent_w);

/* Library, host-only: the same for a given precision (RF_PREC_FP8 adds the e4m3
 * tensors and scales) and a key/value geometry of its own (plan_kv NULL, or
 * S_kv <= 0: the query's; see rf_prepare_ex). */
rf_status_t rf_workspace_layout_ex(rf_precision_t precision, int B, int N, int D, const rf_plan_t* plan,
                                   const rf_plan_t* plan_kv, rf_ws_layout_t* layout);
size_t rf_workspace_size_ex(rf_precision_t precision, int B, int S, int N, int D, int txt_len, int latent_t,
                            int latent_h, int latent_w, int S_kv, int kv_t, int kv_h, int kv_w);

/* The whole rf_v2 call: [SA] sparse_type "rf_v2" (token reorder -> block
 * pooling -> top-k sparse mask -> rain_fusion_attention -> inverse
 * reorder), its parameters scale (NaN or <= 0: head_dim ** -0.5), head_num
 * (N), input_layout, txt_len, block_size, latent_shape_q, sparsity, and
 * "Returns" (out shaped like q); the dense fallbacks of [RF] intro.  Here
 * with a workspace cached by the library per device
 * (grown with cudaMalloc on first use of a larger shape; never shrunk).  The
 * cached buffers are shared by rf_sparse_attention, rf_sparse_attention_ex
 * (NULL workspace) and rf_sparse_attention_host(_ex) on a device: calls from
 * several host threads to the same device must be serialised by the caller,
 * and device calls must be ordered on one stream. */
rf_status_t rf_sparse_attention(const void* q, const void* k, const void* v, rf_layout_t layout, int B, int S, int N,
                                int D, int txt_len, int latent_t, int latent_h, int latent_w, int block_size,
                                float sparsity, float scale, void* out, void* stream);

/* Library: the whole call (as rf_sparse_attention) with a caller-owned device workspace of ws_bytes
 * (>= rf_workspace_size, 256-byte aligned).  Calls that share a workspace
 * must be ordered on one stream.  With a caller-owned workspace a call (this
 * one, rf_sparse_attention_ex, or rf_prepare(_ex) + rf_attend(_ex)) only
 * enqueues kernels and memsets on `stream`, so it can be captured in a CUDA
 * graph and replayed; the graph holds the buffers' addresses.  The cached
 * workspace of rf_sparse_attention may be allocated on first use and is not
 * for capture. */
rf_status_t rf_sparse_attention_ws(const void* q, const void* k, const void* v, rf_layout_t layout, int B, int S,
                                   int N, int D, int txt_len, int latent_t, int latent_h, int latent_w,
                                   int block_size, float sparsity, float scale, void* out, void* workspace,
                                   size_t ws_bytes, void* stream);

/* Stage 1, [SA] pipeline steps one to three (token reorder + block pooling,
 * then block scores + top-k mask), with [RF] intro's forced first-frame
 * blocks:
 * fills q_int/k_int/v_int, pooled_q/pooled_k, mask, kept and margin of the
 * workspace. */
rf_status_t rf_prepare(const void* q, const void* k, const void* v, rf_layout_t layout, int B, int S, int N, int D,
                       int txt_len, int latent_t, int latent_h, int latent_w, int block_size, float sparsity,
                       void* workspace, size_t ws_bytes, void* stream);

/* Stage 2, [SA] pipeline steps four and five (rain_fusion_attention +
 * inverse reorder): attention of every
 * query over its key set as given by the workspace mask, written to out in
 * the caller's token order and layout.  The mask region may be overwritten
 * between the stages (e.g. to run under another mask). */
rf_status_t rf_attend(rf_layout_t layout, int B, int S, int N, int D, int txt_len, int latent_t, int latent_h,
                      int latent_w, int block_size, float sparsity, float scale, void* out, void* workspace,
                      size_t ws_bytes, void* stream);

/* rf_prepare / rf_attend / rf_sparse_attention_ws for any input type ([SA]
 * intro: float16 and bfloat16), precision ([RF] "Configuration": precision)
 * and key/value geometry ([SA] latent_shape_k) (the plain entry points are these with
 * RF_BF16, RF_PREC_NATIVE and S_kv = 0).
 * - Key/value geometry (lite_boost.ops.sparse_attention, latent_shape_k):
 *   S_kv <= 0 means k and v have q's length and geometry (kv_* ignored).
 *   Otherwise k and v hold S_kv = txt_len + kv_t * kv_h * kv_w tokens
 *   (kv latent (0, 0, 0): no geometry) in the same layout, with the same
 *   txt_len: q is reordered and blocked by its geometry, k and v by theirs;
 *   block scores are nb_q x nb_kv, k counts key blocks, the forced columns
 *   are the key geometry's first-frame blocks and the dense rows the query
 *   geometry's, every query attends to the key prefix; if either geometry is
 *   dense (no geometry, or fewer than 32 blocks) the call is dense attention
 *   of every query over every key.  out has q's shape.  The mask region is
 *   [B, N, nb_q, ceil(nb_kv / 32)].
 * - The workspace must come from rf_workspace_size_ex with the same
 *   precision and geometries; rf_sparse_attention_ex takes workspace = NULL
 *   (ws_bytes ignored) to use the library's cached workspace.
 * - Invalid dtype or precision: RF_ERR_ARG.
 * - RF_PREC_FP8 stage 1 writes the reordered q, k, v as e4m3 codes with
 *   their tile scales (q8/k8/v8, scales, vmax) instead of 16-bit copies;
 *   its stage 2 reads only those. */
rf_status_t rf_prepare_ex(const void* q, const void* k, const void* v, rf_dtype_t dtype, rf_precision_t precision,
                          rf_layout_t layout, int B, int S, int N, int D, int txt_len, int latent_t, int latent_h,
                          int latent_w, int S_kv, int kv_t, int kv_h, int kv_w, int block_size, float sparsity,
                          void* workspace, size_t ws_bytes, void* stream);
rf_status_t rf_attend_ex(rf_dtype_t dtype, rf_precision_t precision, rf_layout_t layout, int B, int S, int N, int D,
                         int txt_len, int latent_t, int latent_h, int latent_w, int S_kv, int kv_t, int kv_h,
                         int kv_w, int block_size, float sparsity, float scale, void* out, void* workspace,
                         size_t ws_bytes, void* stream);
rf_status_t rf_sparse_attention_ex(const void* q, const void* k, const void* v, rf_dtype_t dtype,
                                   rf_precision_t precision, rf_layout_t layout, int B, int S, int N, int D,
                                   int txt_len, int latent_t, int latent_h, int latent_w, int S_kv, int kv_t,
                                   int kv_h, int kv_w, int block_size, float sparsity, float scale, void* out,
                                   void* workspace, size_t ws_bytes, void* stream);

/* [SA] pipeline, last step, alone (the inverse reorder, which the attention
 * otherwise fuses into its epilogue): o_int [B, N, S_int, 128] of 16-bit values (internal
 * order) -> out in the caller's layout.  Pad rows are skipped. */
rf_status_t rf_unpermute(const void* o_int, rf_layout_t layout, int B, int S, int N, int D, int txt_len,
                         int latent_t, int latent_h, int latent_w, void* out, void* stream);

/* Library: the whole call (as rf_sparse_attention) end-to-end through HOST
 * buffers (bf16, caller layout): copies q, k, v to
 * the device, runs the call, copies the result back to out_host and
 * synchronises.  The heads are independent, so the call runs on chunks of
 * heads (about 96 MiB of q, k and v each, and at least two heads in BSND) in
 * two device slots: chunk i + 1
 * is copied in and chunk i - 1 copied out, on two library-owned streams,
 * while chunk i computes on its slot's library-owned stream, after the work
 * already queued on `stream` (so that a chunk's kernels can start while the
 * previous chunk's last units still run).  Buffers are cached by the library per
 * device.  Host buffers should be pinned: pageable ones still give the right
 * result, with the copies no longer overlapping the compute.  On return no
 * copy of the caller's buffers is in flight, also after an error. */
rf_status_t rf_sparse_attention_host(const void* q_host, const void* k_host, const void* v_host, rf_layout_t layout,
                                     int B, int S, int N, int D, int txt_len, int latent_t, int latent_h,
                                     int latent_w, int block_size, float sparsity, float scale, void* out_host,
                                     void* stream);
/* Library: rf_sparse_attention_host for any input type, precision and
 * key/value geometry, with the arguments and rules of rf_sparse_attention_ex
 * (host buffers of 16-bit values in the caller's layout; k_host and v_host
 * hold S_kv tokens when S_kv > 0).  The same chunked pipeline: the heads
 * are independent in every precision (an fp8 block scale belongs to one
 * head's tile, vmax to one head), so the result equals the device call on
 * the whole tensors bit for bit.  rf_sparse_attention_host is this with
 * RF_BF16, RF_PREC_NATIVE and S_kv = 0. */
rf_status_t rf_sparse_attention_host_ex(const void* q_host, const void* k_host, const void* v_host, rf_dtype_t dtype,
                                        rf_precision_t precision, rf_layout_t layout, int B, int S, int N, int D,
                                        int txt_len, int latent_t, int latent_h, int latent_w, int S_kv, int kv_t,
                                        int kv_h, int kv_w, int block_size, float sparsity, float scale,
                                        void* out_host, void* stream);

/* Library: synchronises `stream`, reads the workspace status word into *status
 * (0 = fine, otherwise an rf_status_t code recorded by a kernel) and clears
 * it.  The status word sits at the same place in every workspace (any
 * precision or key geometry); the plan only validates the arguments.
 * Returns RF_OK, RF_ERR_ARG, RF_ERR_WORKSPACE or RF_ERR_CUDA. */
rf_status_t rf_read_status(void* workspace, size_t ws_bytes, int B, int N, int D, const rf_plan_t* plan,
                           int* status, void* stream);

/* Library: synchronises `stream` and reads *stats from a workspace after rf_prepare +
 * rf_attend (or rf_sparse_attention_ws) with keys in the query's geometry
 * and native precision: the kept counts and k-th-score margins of the mask,
 * the redo list and the status word (copied, not cleared).  The debug view of
 * a call: how much of the sequence it kept, how many selections sat on a
 * near-tie (k-th and (k+1)-th block scores within 1e-5, relative), how
 * many tiles took the second pass.
 * Returns RF_OK, RF_ERR_ARG, RF_ERR_WORKSPACE or RF_ERR_CUDA. */
rf_status_t rf_read_stats(void* workspace, size_t ws_bytes, int B, int N, int D, const rf_plan_t* plan,
                          rf_stats_t* stats, void* stream);
/* Library: the same after a call of any precision and key/value geometry
 * (rf_prepare_ex + rf_attend_ex, or rf_sparse_attention_ex with a
 * workspace): plan and plan_kv as rf_plan_kv gives them (plan_kv NULL: the
 * query's).  kept_pairs and density then count the key sequence's length:
 * dense rows read all of S_kv keys, a sparse block's rows the key prefix and
 * 128 keys per kept key block. */
rf_status_t rf_read_stats_ex(rf_precision_t precision, void* workspace, size_t ws_bytes, int B, int N, int D,
                             const rf_plan_t* plan, const rf_plan_t* plan_kv, rf_stats_t* stats, void* stream);

/* Library test control of the device-side waits of the attention kernel, process-wide,
 * read at each launch.  wait_limit_ns: limit of every wait (0 = the default,
 * 2 s).  skip_first_q = 1: every CTA's first query tile never gets its Q
 * copy, so the first wait on it runs out; the kernel then records
 * RF_ERR_TIMEOUT in the workspace status word (read with rf_read_status),
 * lets its issued copies land, frees its tensor memory and returns, and the
 * output is not valid.  Used by the tests to exercise the timeout path
 * without any fault; call with (0, 0) to restore normal operation. */
rf_status_t rf_debug_set_wait(long long wait_limit_ns, int skip_first_q);

/* Library test control of the attention path, process-wide, read at each launch.
 * path 0 (default): the three-chain kernel runs every query tile and hands
 * the tiles whose P left the type's headroom to the two-tile kernel; path 1:
 * the two-tile kernel runs every query tile.  sum_limit > 0 replaces the
 * headroom test (a sum of P above it over one softmax task of the chain
 * kernel -- a unit's first tile, then half tiles of 64 keys in 16-bit and
 * whole tiles in fp8 -- hands the query tile on; 0 = the type's own: 2^64
 * for bf16, 65504 for fp16, 448 for e4m3), so a test can send a chosen share
 * of the tiles through the second pass.  Returns RF_ERR_ARG on path outside
 * {0, 1} or sum_limit < 0. */
rf_status_t rf_debug_set_path(int path, float sum_limit);

/* Library measurement hook, process-wide: while `event` is not NULL, rf_prepare /
 * rf_prepare_ex record it (cudaEventRecord) on their stream between the
 * reorder + block-mean kernel (K1) and the kernels after it (block scores +
 * top-k, fp8 quantisation), so a caller's CUDA events around the call can
 * time K1 alone.  `event` is a cudaEvent_t the caller created and keeps
 * alive while it is set; NULL clears the hook.  The library never destroys
 * it.  A failed record is returned by the prepare call as RF_ERR_CUDA. */
rf_status_t rf_debug_set_stage_event(void* event);

/* Size of the library-owned static scratch array of rf_block_mask_noalloc,
 * per device (32 MiB): enough for B * N * nb <= 32768 block rows of pooled Q and K
 * (the 56-head MiniMax-H3 shape needs 26,040). */
#define RF_NOALLOC_SCRATCH_BYTES (32u << 20)

/* Block mask without any device allocation.  The pages have no counterpart:
 * this is a library convenience for callers that cannot allocate device
 * memory themselves.  q and k are bf16 (the only input type it takes).  Examples are a plugin in a process whose device memory
 * belongs entirely to one allocator that forbids side allocations, or a
 * latency-critical loop that cannot afford the implicit synchronisation of
 * cudaMalloc/cudaFree.
 * It computes what rf_prepare puts in the mask, kept and margin regions
 * (block pooling of q and k over the reordered sparse blocks, block scores,
 * top-k plus the forced first-frame blocks) and writes them to the caller's
 * device buffers: mask uint32 [B, N, nb, ceil(nb / 32)], kept int32
 * [B, N, nb], margin fp32 [B, N, nb] (nb and the geometry as in rf_plan).
 * Its only scratch, the fp32 block means of q and k, lives in a file-scope
 * static device array of RF_NOALLOC_SCRATCH_BYTES that every device loading
 * the library holds until the process exits.  It calls no cudaMalloc,
 * cudaFree or allocating routine.
 * - B * N * nb * 128 * 8 bytes above RF_NOALLOC_SCRATCH_BYTES returns
 *   RF_ERR_UNSUPPORTED with a message; a dense plan (nb = 0) writes nothing.
 * - The first call on a device looks up the device address of the array
 *   (cudaGetSymbolAddress) with that device current; make that first call
 *   before any stream capture.  The address is kept per device and CUDA
 *   context: after a device reset (or a new primary context) the next call
 *   looks it up again, and that call too should come before any capture.
 * - All calls share the array: calls whose work overlaps on the GPU race
 *   and must be ordered by the caller.  Each call rewrites all the scratch
 *   it reads, so nothing needs clearing between calls. */
rf_status_t rf_block_mask_noalloc(const void* q, const void* k, rf_layout_t layout, int B, int S, int N, int D,
                                  int txt_len, int latent_t, int latent_h, int latent_w, int block_size,
                                  float sparsity, uint32_t* mask, int32_t* kept, float* margin, void* stream);

/* Library debug kernel: y[i] = 2^x[i] for n fp32 values (device pointers,
 * 4-byte aligned, may be the same array), computed two at a time by the
 * exponential the attention's softmax runs on the FMA pipe for a share of
 * its weights: 2^round(x) by the exponent field times a degree-3 polynomial
 * for 2^f, |f| <= 1/2 (relative error below 7.5e-5).  x is clamped to
 * [-125, 128] first, so x < -125 gives about 2^-125, x >= 127.5 at least
 * 2^127.5 (never a small or negative number: a softmax sum that overflows
 * stays visible as one), and NaN gives about 2^-125.  Asynchronous on
 * `stream`.  Returns RF_ERR_ARG for n < 0, NULL or misaligned pointers. */
rf_status_t rf_debug_exp2_poly(const float* x, float* y, int n, void* stream);

/* Library: thread-local text of the last error returned on this thread. */
const char* rf_last_error_string(void);

#ifdef __cplusplus
}
#endif

#endif /* RFSA_H */
