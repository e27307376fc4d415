// internal.h - host-side entry points shared by the translation units of
// libattn_b200.so (not part of the public C ABI; see include/attn.h).
#pragma once
#include <cuda.h>
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
  // per-head linear distance bias slopes (natural-log units), or null
  const float* slopes = nullptr;
  // key window [i - window_left, i + window_right] around query row i; -1:
  // unbounded on that side (bf16 path only)
  int window_left = -1, window_right = -1;
};

// Fused tcgen05 path (fused_fwd.cu). Arguments already validated.
int launch_fused(const AttnArgs& a, cudaStream_t stream);

// FP8 variant (d = 128): q, k, v hold E4M3 bytes; the attended values are
// q_descale * Q, k_descale * K, v_descale * V. Arguments already validated.
int launch_fused_fp8(const AttnArgs& a, float q_descale, float k_descale, float v_descale,
                     cudaStream_t stream);

// kv path: Nq query rows against Nk keys per head.
struct AttnKvArgs {
  const void* q;
  const void* k;
  const void* v;
  void* o;
  float* lse;
  int B, H, Nq, Nk, d;
  float scale;
  int causal;
  int window_left, window_right;  // key window around the query position; < 0: unbounded
  const float* slopes;            // per-head linear distance bias slopes (device), or null
};

// How the kv path cuts the work: T KV tiles of 128 keys, tps tiles per split,
// nsplit splits (none empty), nqb query blocks per head; alt = 1 when Nq <= 128
// (one query tile per CTA, its two softmax warpgroups on alternate KV tiles).
struct KvPlan {
  int T, tps, nsplit, alt, nqb;
  int t_begin;  // first KV tile any query row needs; the splits cut [t_begin, T)
};

constexpr int kMaxKvSplits = 256;

// Plan for a requested split count (clamped to [1, T - t_begin]); window_left
// < 0 means no left window bound.
KvPlan plan_kv(int BH, int Nq, int Nk, int num_splits, int window_left);
// Split count the library picks for a GPU with `sms` multiprocessors.
int default_kv_splits(int BH, int Nq, int Nk, int sms, int window_left);
// Bytes of the fp32 partial-O block (rounded up to 256) and of the whole
// workspace (partial O, then partial lse) for nsplit splits; 0 when nsplit <= 1.
size_t kv_partial_o_bytes(int BH, int Nq, int d, int nsplit);
size_t kv_workspace_bytes(int BH, int Nq, int d, int nsplit);
// Fused kernel over the plan, then the combine when plan.nsplit > 1.
int launch_fused_kv(const AttnKvArgs& a, const KvPlan& plan, void* workspace, cudaStream_t stream);

// LSE-weighted combine of nsplit partial results (combine.cu): for each of
// `rows` rows, O = sum_s w_s O_s / sum_s w_s with w_s = exp(lse_s - max lse),
// lse = max lse + log sum_s w_s; O written as bf16.
int launch_lse_combine(const float* part_o, const float* part_lse, void* o, float* lse, int rows,
                       int d, int nsplit, cudaStream_t stream);

// Elementwise chain y = act(alpha x + b) (chain.cu): one pass when fused,
// else three passes through tmp. Arguments already validated.
int launch_chain(const void* x, const void* b, void* y, void* tmp, long long rows, int cols,
                 float alpha, int act, bool fused, cudaStream_t stream);

// Unfused three-kernel path (naive.cu). Arguments already validated.
int launch_naive(const AttnArgs& a, void* workspace, cudaStream_t stream);

// Device address of the fixed scratch array used by attn_fwd_naive_noalloc on
// the current device (naive.cu); nullptr if the lookup failed.
void* noalloc_scratch_ptr();

// Limit of every bounded wait in the fused kernels, for launches made from
// now on (fused_fwd.cu); default 2000 ms.
void set_wait_limit_ms(int ms);
int wait_limit_ms();

// Tensor map of a [d2][d1][d0] bf16 array (d0 innermost), box {box0, box1, 1},
// 128-byte swizzle, zero fill out of bounds (fused_fwd.cu).
bool encode_bf16_tiled_3d(CUtensorMap* m, const void* ptr, uint64_t d0, uint64_t d1, uint64_t d2,
                          uint32_t box0, uint32_t box1);
// Address of the device error word in the current context, or null.
unsigned int* library_error_word();

// Device error word of the current device (fused_fwd.cu).
int read_and_clear_device_error(cudaStream_t stream);

// exp2_poly self-test kernel (selftest.cu).
int launch_exp2_poly_selftest(const float* x, float* y, int n, cudaStream_t stream);

// Watchdog self-test kernel (fused_fwd.cu).
int launch_wait_timeout_selftest(int limit_ms, cudaStream_t stream);

}  // namespace attn
