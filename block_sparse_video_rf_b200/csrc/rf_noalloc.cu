// Block mask without any device allocation.
//
// Some callers cannot allocate device memory on their own. Examples: a plugin whose
// host process hands all device memory to one allocator (a serving engine's
// preallocated pool, a framework's caching allocator) and forbids side
// allocations, or a latency-critical loop where the implicit device
// synchronisation of cudaMalloc/cudaFree is not acceptable.  For them this file
// computes the rf_v2 block mask (block pooling of Q and K over the reordered
// sparse blocks, block scores, top-k plus forced first-frame blocks) with its
// only scratch -- the fp32 block means of Q and K -- in a library-owned static
// device array of fixed size.  The caller passes inputs and outputs only.
//
// The static array exists once per device that loads the library and stays
// allocated until the process exits.  Every call shares it: calls whose
// kernels overlap on the GPU (two streams, or two host threads) race on it and
// must be ordered by the caller.  Each call overwrites every element it later
// reads, so nothing has to start at zero and the previous call's contents do
// not matter.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "rf_dtype.h"
#include "rf_geometry.h"
#include "rf_kernels.h"

namespace rf {

namespace {

constexpr size_t kNoAllocScratchBytes = RF_NOALLOC_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kThreads = 256;        // 16 column chunks x 16 rows per pass
constexpr int kRowsPerPass = 16;
constexpr int kPasses = RF_BLOCK / kRowsPerPass;

// One CTA = one sparse block of one (b, head): the fp32 means of its 128 q
// rows and 128 k rows, summed in the same order as the reorder kernel's fused
// pooling (per thread over 8 rows, then over the 16 row groups), so the block
// means -- and hence the mask -- are identical to the ones of rf_prepare.
template <bool kF16>
__global__ void __launch_bounds__(kThreads) pool_blocks_kernel(const uint16_t* __restrict__ q,
                                                               const uint16_t* __restrict__ k, int layout, int B,
                                                               int S, int N, rf_plan_t g, float* __restrict__ pooled_q,
                                                               float* __restrict__ pooled_k) {
  __shared__ float red[2][kRowsPerPass][RF_HEAD_DIM];
  const int blk = blockIdx.x;
  const int bn = blockIdx.y;
  const int b = bn / N, n = bn - b * N;
  const int chunk = threadIdx.x & 15;
  const int rsub = threadIdx.x >> 4;
  const uint16_t* srcs[2] = {q, k};
  const RfBlockTiles bt = rf_block_tiles(g, blk);   // the block's two 8x8 tiles
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int p = 0; p < kPasses; ++p) {
      const int s = rf_src_in_block(g, bt, p * kRowsPerPass + rsub);
      const uint4 u = __ldg(reinterpret_cast<const uint4*>(srcs[t] + rf_token_offset(layout, B, S, N, b, n, s) +
                                                           chunk * 8));
      acc_half8<kF16>(acc, u);
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) red[t][rsub][chunk * 8 + i] = acc[i];
  }
  __syncthreads();
  const int t = threadIdx.x >> 7, c = threadIdx.x & 127;
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < kRowsPerPass; ++i) s += red[t][i][c];
  float* dst = (t == 0 ? pooled_q : pooled_k) + ((int64_t)bn * g.nb + blk) * RF_HEAD_DIM + c;
  *dst = s * (1.0f / RF_BLOCK);
}

// Device address of the static scratch array, resolved once per device and
// CUDA context: a device reset, or a primary context released and made
// again, loads the module anew and may move the array, so the address is
// looked up again whenever the current context is not the one it was taken in.
constexpr int kMaxDevices = 64;
struct ScratchAddr {
  unsigned long long ctx_id;
  void* ptr;
};
std::mutex g_addr_mu;
ScratchAddr g_addr[kMaxDevices] = {};

// Id of the current context (false when there is none yet).  The driver's
// functions are reached through the runtime's entry-point query, so the
// library does not link against the driver library and still loads where
// there is none.
typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

bool current_ctx_id(unsigned long long* id) {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  if (!get_current || !get_id) {
    void* a = nullptr;
    void* b = nullptr;
    cudaDriverEntryPointQueryResult qa, qb;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &a, cudaEnableDefault, &qa) != cudaSuccess ||
        qa != cudaDriverEntryPointSuccess || !a)
      return false;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &b, cudaEnableDefault, &qb) != cudaSuccess ||
        qb != cudaDriverEntryPointSuccess || !b)
      return false;
    get_current = reinterpret_cast<CtxGetCurrentFn>(a);
    get_id = reinterpret_cast<CtxGetIdFn>(b);
  }
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS || !ctx) return false;
  return get_id(ctx, id) == CUDA_SUCCESS;
}

}  // namespace

cudaError_t noalloc_scratch(void** ptr) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_addr_mu);
  unsigned long long id = 0;
  if (g_addr[dev].ptr && current_ctx_id(&id) && id == g_addr[dev].ctx_id) {
    *ptr = g_addr[dev].ptr;
    return cudaSuccess;
  }
  // In host code g_noalloc_scratch names a host-side stand-in; the kernel
  // needs the device address of this device's copy.  The lookup also makes
  // the device's primary context current if no context was.
  void* p = nullptr;
  e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
  if (e != cudaSuccess) return e;
  if (!current_ctx_id(&id)) return cudaErrorDeviceUninitialized;
  g_addr[dev].ctx_id = id;
  g_addr[dev].ptr = p;
  *ptr = p;
  return cudaSuccess;
}

cudaError_t launch_block_mask_noalloc(const void* q, const void* k, int dtype, int layout, int B, int S, int N,
                                      const rf_plan_t& g, uint32_t* mask, int* kept, float* margin,
                                      cudaStream_t stream) {
  void* scratch = nullptr;
  cudaError_t e = noalloc_scratch(&scratch);
  if (e != cudaSuccess) return e;
  float* pooled_q = static_cast<float*>(scratch);
  float* pooled_k = pooled_q + (size_t)B * N * g.nb * RF_HEAD_DIM;
  dim3 grid(g.nb, B * N);
  auto kern = dtype == RF_F16 ? pool_blocks_kernel<true> : pool_blocks_kernel<false>;
  kern<<<grid, kThreads, 0, stream>>>(static_cast<const uint16_t*>(q), static_cast<const uint16_t*>(k), layout, B, S,
                                      N, g, pooled_q, pooled_k);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return launch_mask(pooled_q, pooled_k, B * N, g, g, mask, kept, margin, stream);
}

}  // namespace rf
