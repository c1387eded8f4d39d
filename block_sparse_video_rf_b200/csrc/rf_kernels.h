// Launchers of the library's kernels (internal to the library).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "rfsa.h"

namespace rf {

// K1: token reorder into [B, N, S_int, 128] 16-bit rows for q (query plan g,
// S rows) and k, v (key plan gk, Sk rows; pad rows zeroed), with the fp32
// block means of q and k for the sparse blocks; dtype (rf_dtype_t) says how
// the pooling reads the values.
cudaError_t launch_permute_pool(const void* q, const void* k, const void* v, int dtype, int layout, int B, int S,
                                int Sk, int N, const rf_plan_t& g, const rf_plan_t& gk, void* q_int, void* k_int,
                                void* v_int, float* pooled_q, float* pooled_k, cudaStream_t stream);

// K1 at the fp8 precision (RF_PREC_FP8): the same reorder and block means,
// with the reordered tiles written as e4m3 codes instead of 16-bit rows: per
// (tensor, head, 128-row tile) scale = amax / 448 and codes of x * 448 / amax;
// V's tiles stored transposed; scales = q [BN, g.n_tiles], then k and v
// [BN, gk.n_tiles]; vmax[bn] = the largest V tile scale of head bn (zeroed
// here first).
cudaError_t launch_permute_pool_fp8(const void* q, const void* k, const void* v, int dtype, int layout, int B, int S,
                                    int Sk, int N, const rf_plan_t& g, const rf_plan_t& gk, uint8_t* q8, uint8_t* k8,
                                    uint8_t* v8, float* scales, float* vmax, float* pooled_q, float* pooled_k,
                                    cudaStream_t stream);

// K4: inverse reorder of an internal-order tensor into the caller's layout.
cudaError_t launch_unpermute(const void* o_int, int layout, int B, int S, int N, const rf_plan_t& g, void* out,
                             cudaStream_t stream);

// K2: block scores (g.nb query blocks x gk.nb key blocks) + top-k (gk.k) +
// forced first-frame blocks (key columns gk.ff, query rows g.ff) -> bit mask
// rows, kept counts and k-th-score margins.
cudaError_t launch_mask(const float* pooled_q, const float* pooled_k, int BN, const rf_plan_t& g,
                        const rf_plan_t& gk, uint32_t* mask, int* kept, float* margin, cudaStream_t stream);

// Test controls of the attention kernel's bounded waits (see rf_debug_set_wait).
struct AttnDebug {
  long long wait_limit_ns = 0;   // 0: the default limit (2 s)
  int skip_first_q = 0;          // 1: the first unit of every CTA never gets its Q tile
  int path = 0;                  // 16-bit: 0 chain_kernel then the second pass; 1 attn_kernel over every unit
  float sum_limit = 0.f;         // chain_kernel: tile sum of P that hands a unit on (0: the P type's headroom)
};

// K3, 16-bit: block-sparse flash attention over the internal layout, output
// written straight to the caller's layout (inverse reorder fused in the
// epilogue).  Operands and output in dtype (rf_dtype_t).  chain_kernel runs
// every unit and lists in `redo` ([0] a work counter, [1] a count, [2 ...]
// unit ids; 2 + B*N*g.n_tiles ints) those whose P left the type's headroom;
// attn_kernel then computes the listed units.
cudaError_t launch_attention(const void* q_int, const void* k_int, const void* v_int, const uint32_t* mask,
                             int dtype, int layout, int B, int S, int N, const rf_plan_t& g, const rf_plan_t& gk,
                             float scale, void* out, int* counter, int* status, int* redo, const AttnDebug& dbg,
                             cudaStream_t stream);

// attn_kernel (two query tiles per CTA, running maximum with rescaling) over
// every unit (list_mode 0) or over the units listed in `redo` (list_mode 1).
cudaError_t launch_attention_slots(const void* q_int, const void* k_int, const void* v_int, const uint32_t* mask,
                                   int dtype, int layout, int B, int S, int N, const rf_plan_t& g,
                                   const rf_plan_t& gk, float scale, void* out, int* counter, int* status, int* redo,
                                   int list_mode, const AttnDebug& dbg, cudaStream_t stream);

// K3 on the e4m3 tensors of launch_permute_pool_fp8; output in dtype.  As
// launch_attention: chain_kernel, then attn_kernel over the units it lists
// (P above e4m3's 448).
cudaError_t launch_attention_fp8(const uint8_t* q8, const uint8_t* k8, const uint8_t* v8, const float* scales,
                                 const float* vmax, const uint32_t* mask, int dtype, int layout, int B, int S, int N,
                                 const rf_plan_t& g, const rf_plan_t& gk, float scale, void* out, int* counter,
                                 int* status, int* redo, const AttnDebug& dbg, cudaStream_t stream);
// attn_kernel's fp8 form over every unit (list_mode 0) or the units listed in redo (list_mode 1).
cudaError_t launch_attention_fp8_slots(const uint8_t* q8, const uint8_t* k8, const uint8_t* v8, const float* scales,
                                       const float* vmax, const uint32_t* mask, int dtype, int layout, int B, int S,
                                       int N, const rf_plan_t& g, const rf_plan_t& gk, float scale, void* out,
                                       int* counter, int* status, int* redo, int list_mode, const AttnDebug& dbg,
                                       cudaStream_t stream);

// Block mask with the pooled means in the library's static scratch array
// (no device allocation); see rf_block_mask_noalloc.
cudaError_t launch_block_mask_noalloc(const void* q, const void* k, int dtype, int layout, int B, int S, int N,
                                      const rf_plan_t& g, uint32_t* mask, int* kept, float* margin,
                                      cudaStream_t stream);

// Debug: the attention's FMA-pipe exponential (exp2_poly_x2) on n fp32
// values, y[i] = 2^x[i] as the softmax computes it.
cudaError_t launch_debug_exp2_poly(const float* x, float* y, int n, cudaStream_t stream);

}  // namespace rf
