// chain.cu - elementwise chain y = act(alpha * x + b), fused (one pass over
// HBM) and unfused (three passes), declared in include/chain.h.
//
// Both are HBM-bound streams: 16-byte vector loads and stores (eight bf16
// per thread per step), a grid-stride loop over a grid of a few CTAs per SM,
// so every SM keeps enough bytes in flight to saturate the memory system.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include "../../include/chain.h"
#include "internal.h"

namespace attn {
namespace {

constexpr int kThreadsPerBlock = 256;
constexpr int kBlocksPerSm = 8;

__device__ __forceinline__ float act_of(float z, int act) {
  switch (act) {
    case CHAIN_ACT_RELU: return fmaxf(z, 0.0f);
    case CHAIN_ACT_GELU: return 0.5f * z * (1.0f + erff(z * 0.70710678118654752f));
    default: return z / (1.0f + __expf(-z));
  }
}

__device__ __forceinline__ void unpack8(const uint4& u, float (&f)[8]) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 p = __bfloat1622float2(h[i]);
    f[2 * i] = p.x;
    f[2 * i + 1] = p.y;
  }
}

__device__ __forceinline__ uint4 pack8(const float (&f)[8]) {
  uint4 u;
  __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
  return u;
}

// Stage selector of the generic pass: which of the three steps it applies.
enum Stage : int { kScale = 1, kBias = 2, kAct = 4 };

// One pass over n8 vectors of eight elements: applies the stages in `stages`
// (the fused kernel passes all three, the unfused path one per launch). in and
// out may be the same array (the unfused bias pass works in place): each
// thread reads an element before it writes it and no two threads share one.
__global__ void __launch_bounds__(kThreadsPerBlock)
    chain_pass_kernel(const uint4* in, const uint4* __restrict__ bias, uint4* out, long long n8,
                      int cols8, float alpha, int act, int stages) {
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < n8;
       i += stride) {
    float v[8];
    unpack8(in[i], v);
    if (stages & kScale) {
#pragma unroll
      for (int e = 0; e < 8; ++e) v[e] *= alpha;
    }
    if (stages & kBias) {
      float bv[8];
      unpack8(bias[i % cols8], bv);
#pragma unroll
      for (int e = 0; e < 8; ++e) v[e] += bv[e];
    }
    if (stages & kAct) {
#pragma unroll
      for (int e = 0; e < 8; ++e) v[e] = act_of(v[e], act);
    }
    out[i] = pack8(v);
  }
}

int launch_pass(const void* in, const void* bias, void* out, long long n8, int cols8, float alpha,
                int act, int stages, cudaStream_t stream) {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms < 1)
    return ATTN_ERR_CUDA;
  const long long want = (n8 + kThreadsPerBlock - 1) / kThreadsPerBlock;
  const long long cap = static_cast<long long>(sms) * kBlocksPerSm;
  const unsigned grid = static_cast<unsigned>(want < cap ? want : cap);
  chain_pass_kernel<<<grid, kThreadsPerBlock, 0, stream>>>(
      static_cast<const uint4*>(in), static_cast<const uint4*>(bias), static_cast<uint4*>(out), n8,
      cols8, alpha, act, stages);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_LAUNCH;
}

}  // namespace

int launch_chain(const void* x, const void* b, void* y, void* tmp, long long rows, int cols,
                 float alpha, int act, bool fused, cudaStream_t stream) {
  const long long n8 = rows * (cols / 8);
  const int cols8 = cols / 8;
  if (fused) return launch_pass(x, b, y, n8, cols8, alpha, act, kScale | kBias | kAct, stream);
  int st = launch_pass(x, b, tmp, n8, cols8, alpha, act, kScale, stream);
  if (st == ATTN_OK) st = launch_pass(tmp, b, tmp, n8, cols8, alpha, act, kBias, stream);
  if (st == ATTN_OK) st = launch_pass(tmp, b, y, n8, cols8, alpha, act, kAct, stream);
  return st;
}

}  // namespace attn
