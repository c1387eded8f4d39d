// Debug kernels: the attention's building blocks run alone on plain arrays,
// so that tests can check them against their definitions.
//
// exp2_poly_kernel applies the FMA-pipe exponential that the attention uses
// for a share of its softmax weights (exp2_poly_x2 in sm100_ptx.cuh: 2^x
// split into 2^round(x) by the exponent field and 2^f, |f| <= 1/2, by a
// degree-3 polynomial) to an array of fp32 values, two at a time as the
// softmax does.
#include <cuda_runtime.h>

#include "rf_kernels.h"
#include "sm100_ptx.cuh"

namespace rf {

namespace {

__global__ void exp2_poly_kernel(const float* __restrict__ x, float* __restrict__ y, int n) {
  const int pairs = (n + 1) / 2;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < pairs; i += gridDim.x * blockDim.x) {
    const int a = 2 * i, b = 2 * i + 1;
    const float x0 = x[a];
    const float x1 = b < n ? x[b] : 0.f;
    float y0, y1;
    f2_unpack(exp2_poly_x2(f2_pack(x0, x1)), y0, y1);
    y[a] = y0;
    if (b < n) y[b] = y1;
  }
}

}  // namespace

cudaError_t launch_debug_exp2_poly(const float* x, float* y, int n, cudaStream_t stream) {
  if (n <= 0) return cudaSuccess;
  const int pairs = (n + 1) / 2;
  const int threads = 256;
  const int blocks = (pairs + threads - 1) / threads < 4096 ? (pairs + threads - 1) / threads : 4096;
  exp2_poly_kernel<<<blocks, threads, 0, stream>>>(x, y, n);
  return cudaGetLastError();
}

}  // namespace rf
