// combine.cu - LSE-weighted combination of the split-KV partial results.
//
// When the keys of one head are split into ranges that different CTAs attend
// to, split s leaves, for every query row, the normalised partial output O_s
// (softmax over its own keys only) and its log-sum-exp lse_s. Because
// exp(lse_s) is the sum of exp(score) over split s's keys, the softmax over
// all keys is the mixture of the splits with weights exp(lse_s) / sum exp(lse):
//   m = max_s lse_s,  w_s = exp(lse_s - m),  O = sum_s w_s O_s / sum_s w_s,
//   lse = m + log sum_s w_s.
// The article pratikdhanave.com, "The Attention Bottleneck - and How
// FlashAttention Fixed It" ("Key takeaways": context grown from 2K to 128K
// makes attention the dominant long-context cost of inference) motivates the
// shape but describes no splitting of the keys; the identity above is
// elementary algebra on the softmax definition. One warp per row; lane l owns d/32 consecutive columns.
// HBM-bound: nsplit * (d + 1) fp32 reads and 2d + 4 bytes of writes per row.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include "../../include/attn.h"
#include "internal.h"
#include "sm100.cuh"

namespace attn {
namespace {

constexpr int kRowsPerBlock = 8;

template <int D>
__global__ void
    lse_combine_kernel(const float* __restrict__ part_o, const float* __restrict__ part_lse,
                       __nv_bfloat16* __restrict__ o, float* __restrict__ lse, int rows,
                       int nsplit) {
  constexpr int kPer = D / 32;  // columns per lane: 4 (d = 128) or 2 (d = 64)
  const int row = blockIdx.x * kRowsPerBlock + threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  if (row >= rows) return;

  float m = -INFINITY;
  for (int s = lane; s < nsplit; s += 32) m = fmaxf(m, part_lse[static_cast<size_t>(s) * rows + row]);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));

  float acc[kPer];
#pragma unroll
  for (int c = 0; c < kPer; ++c) acc[c] = 0.0f;
  float wsum = 0.0f;
  for (int s0 = 0; s0 < nsplit; s0 += 32) {
    const int s = s0 + lane;
    const float ls = s < nsplit ? part_lse[static_cast<size_t>(s) * rows + row] : -INFINITY;
    const float w = (ls == -INFINITY) ? 0.0f : __expf(ls - m);
    wsum += w;
    const int cnt = min(32, nsplit - s0);
#pragma unroll 4
    for (int t = 0; t < cnt; ++t) {
      const float wt = __shfl_sync(0xffffffffu, w, t);
      const float* src = part_o + (static_cast<size_t>(s0 + t) * rows + row) * D + lane * kPer;
      if constexpr (kPer == 4) {
        const float4 x = *reinterpret_cast<const float4*>(src);
        acc[0] = fmaf(wt, x.x, acc[0]);
        acc[1] = fmaf(wt, x.y, acc[1]);
        acc[2] = fmaf(wt, x.z, acc[2]);
        acc[3] = fmaf(wt, x.w, acc[3]);
      } else {
        const float2 x = *reinterpret_cast<const float2*>(src);
        acc[0] = fmaf(wt, x.x, acc[0]);
        acc[1] = fmaf(wt, x.y, acc[1]);
      }
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) wsum += __shfl_xor_sync(0xffffffffu, wsum, off);

  const float inv = wsum > 0.0f ? 1.0f / wsum : 0.0f;
  __nv_bfloat16* dst = o + static_cast<size_t>(row) * D + lane * kPer;
  if constexpr (kPer == 4) {
    *reinterpret_cast<uint2*>(dst) =
        make_uint2(pack_bf16x2(acc[0] * inv, acc[1] * inv), pack_bf16x2(acc[2] * inv, acc[3] * inv));
  } else {
    *reinterpret_cast<uint32_t*>(dst) = pack_bf16x2(acc[0] * inv, acc[1] * inv);
  }
  if (lane == 0) lse[row] = wsum > 0.0f ? m + __logf(wsum) : -INFINITY;
}

}  // namespace

int launch_lse_combine(const float* part_o, const float* part_lse, void* o, float* lse, int rows,
                       int d, int nsplit, cudaStream_t stream) {
  if (rows <= 0) return ATTN_OK;
  const unsigned grid = static_cast<unsigned>((rows + kRowsPerBlock - 1) / kRowsPerBlock);
  auto* out = static_cast<__nv_bfloat16*>(o);
  if (d == 128)
    lse_combine_kernel<128><<<grid, 32 * kRowsPerBlock, 0, stream>>>(part_o, part_lse, out, lse, rows, nsplit);
  else
    lse_combine_kernel<64><<<grid, 32 * kRowsPerBlock, 0, stream>>>(part_o, part_lse, out, lse, rows, nsplit);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_LAUNCH;
}

}  // namespace attn
