// chain.cu - elementwise chain y = act(alpha * x + b), fused (one pass over
// HBM) and unfused (three passes), declared in include/chain.h.
//
// Both are HBM-bound streams: 16-byte vector loads and stores (eight bf16
// per vector, two vectors per thread and step), a grid-stride loop over one
// wave of resident CTAs, so every SM keeps enough bytes in flight to saturate
// the memory system.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include "../../include/chain.h"
#include "internal.h"
#include "sm100.cuh"

namespace attn {
namespace {

constexpr int kThreadsPerBlock = 256;

// ReLU, GELU (exact normal CDF) and SiLU; the tanh form of GELU is
// gelu_tanh_pair: (1 + tanh u) / 2 = 1 / (1 + e^(-2u)), so it is computed as
// z / (1 + e^(-2u)), free of the cancellation that 1 + tanh u suffers for
// negative z.
__device__ __forceinline__ float act_of(float z, int act) {
  switch (act) {
    case CHAIN_ACT_RELU: return fmaxf(z, 0.0f);
    case CHAIN_ACT_GELU: return 0.5f * z * (1.0f + erff(z * 0.70710678118654752f));
    default: return z / (1.0f + __expf(-z));  // SiLU
  }
}

__device__ __forceinline__ float rcp_approx(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// GELU (tanh form) of a pair in packed f32x2 arithmetic: y = z / (1 + 2^t)
// with t = -2 sqrt(2/pi) log2(e) (z + 0.044715 z^3); two MUFU operations
// (2^t, reciprocal) per element.
__device__ __forceinline__ void gelu_tanh_pair(float& a, float& b) {
  const uint64_t zero = f2_pack(0.0f, 0.0f);
  const uint64_t z = f2_pack(a, b);
  const uint64_t zz = f2_fma(z, z, zero);
  const uint64_t poly = f2_fma(zz, f2_pack(0.044715f, 0.044715f), f2_pack(1.0f, 1.0f));
  const uint64_t t = f2_fma(f2_fma(poly, z, zero), f2_pack(-2.3022082f, -2.3022082f), zero);
  float t0, t1;
  f2_unpack(t, t0, t1);
  const uint64_t den = f2_add(f2_pack(ex2_approx(t0), ex2_approx(t1)), f2_pack(1.0f, 1.0f));
  float d0, d1;
  f2_unpack(den, d0, d1);
  f2_unpack(f2_fma(z, f2_pack(rcp_approx(d0), rcp_approx(d1)), zero), a, b);
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
  // two independent 16-byte loads per thread and step keep enough bytes in
  // flight per SM to cover the memory latency. The bias column of vector i is
  // i mod cols8, tracked by adding the stride's remainder (one 64-bit modulo
  // per thread instead of one per vector).
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  const int step = static_cast<int>(stride % cols8);
  long long i0 = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  int col = static_cast<int>(i0 % cols8);
  for (; i0 < n8; i0 += 2 * stride) {
    uint4 raw[2];
    int cols_of[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const long long i = i0 + h * stride;
      cols_of[h] = col;
      col += step;
      if (col >= cols8) col -= cols8;
      if (i < n8) raw[h] = in[i];
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const long long i = i0 + h * stride;
      if (i >= n8) break;
      float v[8];
      unpack8(raw[h], v);
      if (stages & kScale) {
#pragma unroll
        for (int e = 0; e < 8; ++e) v[e] *= alpha;
      }
      if (stages & kBias) {
        float bv[8];
        unpack8(bias[cols_of[h]], bv);
#pragma unroll
        for (int e = 0; e < 8; ++e) v[e] += bv[e];
      }
      if (stages & kAct) {
        if (act == CHAIN_ACT_GELU_TANH) {
#pragma unroll
          for (int e = 0; e < 8; e += 2) gelu_tanh_pair(v[e], v[e + 1]);
        } else {
#pragma unroll
          for (int e = 0; e < 8; ++e) v[e] = act_of(v[e], act);
        }
      }
      out[i] = pack8(v);
    }
  }
}

int launch_pass(const void* in, const void* bias, void* out, long long n8, int cols8, float alpha,
                int act, int stages, cudaStream_t stream) {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms < 1)
    return ATTN_ERR_CUDA;
  // exactly the CTAs that can be resident at once: a grid-stride loop over a
  // single wave, so no CTA waits for a slot and none finishes late
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, chain_pass_kernel, kThreadsPerBlock,
                                                    0) != cudaSuccess ||
      per_sm < 1)
    return ATTN_ERR_CUDA;
  const long long want = (n8 + 2ll * kThreadsPerBlock - 1) / (2ll * kThreadsPerBlock);
  const long long cap = static_cast<long long>(sms) * per_sm;
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
