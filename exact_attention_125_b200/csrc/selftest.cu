// selftest.cu - device-side numerics checks exposed through the C ABI.
#include <cuda_runtime.h>

#include "../../include/attn.h"
#include "internal.h"
#include "sm100.cuh"

namespace attn {
namespace {

// Evaluates exp2_poly_pair (the FMA-pipe exponential of the fused kernel's
// softmax) on n floats.
__global__ void exp2_poly_selftest_kernel(const float* __restrict__ x, float* __restrict__ y,
                                          int n) {
  const int i0 = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
  if (i0 >= n) return;
  const float a = x[i0];
  const float b = (i0 + 1 < n) ? x[i0 + 1] : 0.0f;
  float pa, pb;
  exp2_poly_pair(a, b, pa, pb);
  y[i0] = pa;
  if (i0 + 1 < n) y[i0 + 1] = pb;
}

}  // namespace

int launch_exp2_poly_selftest(const float* x, float* y, int n, cudaStream_t stream) {
  const int pairs = (n + 1) / 2;
  exp2_poly_selftest_kernel<<<(pairs + 255) / 256, 256, 0, stream>>>(x, y, n);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_LAUNCH;
}

}  // namespace attn
