// internal.h - host-side entry points shared by the translation units of
// libattn_b200.so (not part of the public C ABI; see include/attn.h).
#pragma once
#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>

namespace attn {

struct AttnArgs {
  const void* q;
  const void* k;
  const void* v;
  void* o;
  float* lse;
  int B, H, N, d;
  float scale;
  int causal;
};

// Fused tcgen05 path (fused_fwd.cu). Arguments already validated.
int launch_fused(const AttnArgs& a, cudaStream_t stream);

// Unfused three-kernel path (naive.cu). Arguments already validated.
int launch_naive(const AttnArgs& a, void* workspace, cudaStream_t stream);

// Device address of the fixed scratch array used by attn_fwd_naive_noalloc on
// the current device (naive.cu); nullptr if the lookup failed.
void* noalloc_scratch_ptr();

// Device error word of the current device (fused_fwd.cu).
int read_and_clear_device_error(cudaStream_t stream);

// exp2_poly self-test kernel (selftest.cu).
int launch_exp2_poly_selftest(const float* x, float* y, int n, cudaStream_t stream);

// Watchdog self-test kernel (fused_fwd.cu).
int launch_wait_timeout_selftest(int limit_ms, cudaStream_t stream);

}  // namespace attn
