// api.cu - the C ABI of libattn_b200.so (declared in include/attn.h):
// argument validation, device check, dispatch to the fused or naive path.
#include <cuda_runtime.h>

#include <climits>
#include <cmath>
#include <cstdint>
#include <mutex>

#include "../../include/attn.h"
#include "../../include/chain.h"
#include "ctx_cache.h"
#include "internal.h"

namespace {

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int validate(const void* q, const void* k, const void* v, const void* o, const float* lse, int B,
             int H, int N, int d, float scale, int causal) {
  if (!q || !k || !v || !o || !lse) return ATTN_ERR_NULL;
  if (B < 1 || H < 1 || N < 1) return ATTN_ERR_SHAPE;
  if (static_cast<long long>(B) * H * N > INT_MAX) return ATTN_ERR_SHAPE;
  if (d != 64 && d != 128) return ATTN_ERR_HEADDIM;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) ||
      !aligned(lse, 4))
    return ATTN_ERR_ALIGN;
  if (!std::isfinite(scale)) return ATTN_ERR_SCALE;
  if (causal != 0 && causal != 1) return ATTN_ERR_CAUSAL;
  return ATTN_OK;
}

// sm_100 check of the current device, cached per device ordinal.
int check_device() {
  static int state[64] = {0};  // 0 unknown, 1 ok, -1 unsupported
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return ATTN_ERR_CUDA;
  if (dev < 0 || dev >= 64) return ATTN_ERR_UNSUPPORTED_DEVICE;
  std::lock_guard<std::mutex> lock(mu);
  if (state[dev] == 0) {
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
      return ATTN_ERR_CUDA;
    state[dev] = (major == 10 && minor == 0) ? 1 : -1;
  }
  return state[dev] == 1 ? ATTN_OK : ATTN_ERR_UNSUPPORTED_DEVICE;
}

attn::AttnArgs pack(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
                    int N, int d, float scale, int causal) {
  attn::AttnArgs a;
  a.q = q;
  a.k = k;
  a.v = v;
  a.o = o;
  a.lse = lse;
  a.B = B;
  a.H = H;
  a.N = N;
  a.d = d;
  a.scale = scale;
  a.causal = causal;
  return a;
}

// Multiprocessors of the current device, cached per context.
int sm_count_cached() {
  static attn::CtxCache<int> cache;
  int n = 0;
  if (!cache.get(&n, [](int* out) {
        int dev = 0;
        return cudaGetDevice(&dev) == cudaSuccess &&
               cudaDeviceGetAttribute(out, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess;
      }))
    return 0;
  return n;
}

// A square problem whose 256-row work units would fill at most half of the
// SMs runs as one 128-row query tile per CTA, the layout the split-KV kernel
// uses for short query ranges: the tile's two softmax warpgroups take
// alternate KV tiles and merge their (O, m, l) at the end. Twice the CTAs,
// each with half the KV steps, one launch and no workspace.
bool small_square(int B, int H, int N) {
  const int sms = sm_count_cached();
  const long long units = static_cast<long long>(B) * H * ((N + 255) / 256);
  return sms > 0 && 2 * units <= sms;
}

attn::KvPlan query_tile_plan(int N) {
  attn::KvPlan pl{};
  pl.T = (N + 127) / 128;
  pl.tps = pl.T;
  pl.nsplit = 1;
  pl.alt = 1;
  pl.nqb = pl.T;
  pl.t_begin = 0;
  return pl;
}

}  // namespace

extern "C" {

int attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
             int N, int d, float scale, int causal, attn_stream_t stream) {
  int st = validate(q, k, v, o, lse, B, H, N, d, scale, causal);
  if (st != ATTN_OK) return st;
  if ((st = check_device()) != ATTN_OK) return st;
  if (small_square(B, H, N)) {
    attn::AttnKvArgs a{q, k, v, o, lse, B, H, N, N, d, scale, causal, -1, -1, nullptr};
    return attn::launch_fused_kv(a, query_tile_plan(N), nullptr,
                                 reinterpret_cast<cudaStream_t>(stream));
  }
  return attn::launch_fused(pack(q, k, v, o, lse, B, H, N, d, scale, causal),
                            reinterpret_cast<cudaStream_t>(stream));
}

namespace {

int validate_kv(const void* q, const void* k, const void* v, const void* o, const float* lse,
                int B, int H, int Nq, int Nk, int d, float scale, int causal) {
  if (!q || !k || !v || !o || !lse) return ATTN_ERR_NULL;
  if (B < 1 || H < 1 || Nq < 1 || Nk < 1) return ATTN_ERR_SHAPE;
  if (static_cast<long long>(B) * H * Nq > INT_MAX || static_cast<long long>(B) * H * Nk > INT_MAX)
    return ATTN_ERR_SHAPE;
  if (d != 64 && d != 128) return ATTN_ERR_HEADDIM;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) ||
      !aligned(lse, 4))
    return ATTN_ERR_ALIGN;
  if (!std::isfinite(scale)) return ATTN_ERR_SCALE;
  if (causal != 0 && causal != 1) return ATTN_ERR_CAUSAL;
  if (causal && Nq > Nk) return ATTN_ERR_SHAPE;
  return ATTN_OK;
}

bool kv_shape_ok(int B, int H, int Nq, int Nk, int d) {
  return B >= 1 && H >= 1 && Nq >= 1 && Nk >= 1 && (d == 64 || d == 128) &&
         static_cast<long long>(B) * H * Nq <= INT_MAX && static_cast<long long>(B) * H * Nk <= INT_MAX;
}

int sm_count(int* sms) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return ATTN_ERR_CUDA;
  if (cudaDeviceGetAttribute(sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return ATTN_ERR_CUDA;
  return ATTN_OK;
}

// Requested split count -> effective plan; num_splits = 0 asks for the
// automatic choice on the current device.
int resolve_kv_plan(int B, int H, int Nq, int Nk, int num_splits, int window_left,
                    attn::KvPlan* plan) {
  if (num_splits < 0 || num_splits > attn::kMaxKvSplits) return ATTN_ERR_SHAPE;
  const int BH = B * H;
  if (num_splits == 0) {
    int st = check_device();
    if (st != ATTN_OK) return st;
    int sms = 0;
    if ((st = sm_count(&sms)) != ATTN_OK) return st;
    num_splits = attn::default_kv_splits(BH, Nq, Nk, sms, window_left);
  }
  *plan = attn::plan_kv(BH, Nq, Nk, num_splits, window_left);
  return ATTN_OK;
}

int fwd_ext(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
            int Nq, int Nk, int d, float scale, int causal, int window_left, int window_right,
            const float* slopes, int num_splits, void* workspace, size_t workspace_bytes,
            attn_stream_t stream) {
  int st = validate_kv(q, k, v, o, lse, B, H, Nq, Nk, d, scale, causal);
  if (st != ATTN_OK) return st;
  if (window_left < -1 || window_right < -1) return ATTN_ERR_WINDOW;
  if (slopes && !aligned(slopes, 4)) return ATTN_ERR_ALIGN;
  if (num_splits < 0 || num_splits > attn::kMaxKvSplits) return ATTN_ERR_SHAPE;
  // An explicit split count is checked against the workspace before the
  // device is touched; the automatic one needs the device's SM count.
  if (num_splits == 0 && (st = check_device()) != ATTN_OK) return st;
  attn::KvPlan plan{};
  if ((st = resolve_kv_plan(B, H, Nq, Nk, num_splits, window_left, &plan)) != ATTN_OK) return st;
  const size_t need = attn::kv_workspace_bytes(B * H, Nq, d, plan.nsplit);
  if (need > 0) {
    if (!workspace) return ATTN_ERR_NULL;
    if (!aligned(workspace, 256)) return ATTN_ERR_ALIGN;
    if (workspace_bytes < need) return ATTN_ERR_WORKSPACE;
  }
  if ((st = check_device()) != ATTN_OK) return st;
  attn::AttnKvArgs a;
  a.q = q;
  a.k = k;
  a.v = v;
  a.o = o;
  a.lse = lse;
  a.B = B;
  a.H = H;
  a.Nq = Nq;
  a.Nk = Nk;
  a.d = d;
  a.scale = scale;
  a.causal = causal;
  a.window_left = window_left;
  a.window_right = window_right;
  a.slopes = slopes;
  if (Nq == Nk && plan.nsplit == 1 && small_square(B, H, Nq))
    return attn::launch_fused_kv(a, query_tile_plan(Nq), nullptr,
                                 reinterpret_cast<cudaStream_t>(stream));
  if (Nq == Nk && plan.nsplit == 1) {
    // the square problem, unsplit: the persistent square kernel, which takes
    // the key windows and the distance bias too (the workspace stays unused)
    attn::AttnArgs s;
    s.q = q;
    s.k = k;
    s.v = v;
    s.o = o;
    s.lse = lse;
    s.B = B;
    s.H = H;
    s.N = Nq;
    s.d = d;
    s.scale = scale;
    s.causal = causal;
    s.slopes = slopes;
    s.window_left = window_left;
    s.window_right = window_right;
    return attn::launch_fused(s, reinterpret_cast<cudaStream_t>(stream));
  }
  return attn::launch_fused_kv(a, plan, workspace, reinterpret_cast<cudaStream_t>(stream));
}

int ext_num_splits(int B, int H, int Nq, int Nk, int d, int window_left) {
  if (!kv_shape_ok(B, H, Nq, Nk, d) || window_left < -1) return ATTN_ERR_SHAPE;
  attn::KvPlan plan{};
  const int st = resolve_kv_plan(B, H, Nq, Nk, 0, window_left, &plan);
  return st != ATTN_OK ? st : plan.nsplit;
}

size_t ext_workspace_bytes(int B, int H, int Nq, int Nk, int d, int window_left,
                           int num_splits) {
  if (!kv_shape_ok(B, H, Nq, Nk, d) || window_left < -1) return 0;
  attn::KvPlan plan{};
  if (resolve_kv_plan(B, H, Nq, Nk, num_splits, window_left, &plan) != ATTN_OK) return 0;
  return attn::kv_workspace_bytes(B * H, Nq, d, plan.nsplit);
}

}  // namespace

int attn_fwd_kv(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
                int Nq, int Nk, int d, float scale, int causal, int num_splits, void* workspace,
                size_t workspace_bytes, attn_stream_t stream) {
  return fwd_ext(q, k, v, o, lse, B, H, Nq, Nk, d, scale, causal, -1, -1, nullptr, num_splits,
                 workspace, workspace_bytes, stream);
}

int attn_fwd_kv_num_splits(int B, int H, int Nq, int Nk, int d) {
  return ext_num_splits(B, H, Nq, Nk, d, -1);
}

size_t attn_fwd_kv_workspace_bytes(int B, int H, int Nq, int Nk, int d, int num_splits) {
  return ext_workspace_bytes(B, H, Nq, Nk, d, -1, num_splits);
}

int attn_fwd_ext(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
                 int Nq, int Nk, int d, float scale, int causal, int window_left,
                 int window_right, const float* alibi_slopes, int num_splits, void* workspace,
                 size_t workspace_bytes, attn_stream_t stream) {
  return fwd_ext(q, k, v, o, lse, B, H, Nq, Nk, d, scale, causal, window_left, window_right,
                 alibi_slopes, num_splits, workspace, workspace_bytes, stream);
}

int attn_fwd_ext_num_splits(int B, int H, int Nq, int Nk, int d, int window_left) {
  return ext_num_splits(B, H, Nq, Nk, d, window_left);
}

size_t attn_fwd_ext_workspace_bytes(int B, int H, int Nq, int Nk, int d, int window_left,
                                    int num_splits) {
  return ext_workspace_bytes(B, H, Nq, Nk, d, window_left, num_splits);
}

int attn_fwd_fp8(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
                 int N, int d, float scale, float q_descale, float k_descale, float v_descale,
                 int causal, attn_stream_t stream) {
  int st = validate(q, k, v, o, lse, B, H, N, d, scale, causal);
  if (st != ATTN_OK) return st;
  if (d != 128) return ATTN_ERR_HEADDIM;
  for (float s : {q_descale, k_descale, v_descale})
    if (!std::isfinite(s) || !(s > 0.0f)) return ATTN_ERR_SCALE;
  if ((st = check_device()) != ATTN_OK) return st;
  return attn::launch_fused_fp8(pack(q, k, v, o, lse, B, H, N, d, scale, causal), q_descale,
                                k_descale, v_descale, reinterpret_cast<cudaStream_t>(stream));
}

size_t attn_fwd_naive_workspace_bytes(int B, int H, int N) {
  if (B < 1 || H < 1 || N < 1) return 0;
  const unsigned long long bh = static_cast<unsigned long long>(B) * H;
  const unsigned long long nn = static_cast<unsigned long long>(N) * N;
  if (bh > (1ull << 31) || nn > (1ull << 40)) return 0;
  const unsigned long long elems = bh * nn;
  if (elems > (~0ull) / 4) return 0;
  return static_cast<size_t>(elems * 4ull);  // S and P, bf16 each
}

int attn_fwd_naive(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
                   int N, int d, float scale, int causal, void* workspace, size_t workspace_bytes,
                   attn_stream_t stream) {
  int st = validate(q, k, v, o, lse, B, H, N, d, scale, causal);
  if (st != ATTN_OK) return st;
  if (N > 32768 || static_cast<long long>(B) * H > 65535) return ATTN_ERR_SHAPE;
  if (!workspace) return ATTN_ERR_NULL;
  if (!aligned(workspace, 16)) return ATTN_ERR_ALIGN;
  const size_t need = attn_fwd_naive_workspace_bytes(B, H, N);
  if (need == 0 || workspace_bytes < need) return ATTN_ERR_WORKSPACE;
  if ((st = check_device()) != ATTN_OK) return st;
  return attn::launch_naive(pack(q, k, v, o, lse, B, H, N, d, scale, causal), workspace,
                            reinterpret_cast<cudaStream_t>(stream));
}

int attn_fwd_naive_noalloc(const void* q, const void* k, const void* v, void* o, float* lse,
                           int B, int H, int N, int d, float scale, int causal,
                           attn_stream_t stream) {
  int st = validate(q, k, v, o, lse, B, H, N, d, scale, causal);
  if (st != ATTN_OK) return st;
  if (N > 32768 || static_cast<long long>(B) * H > 65535) return ATTN_ERR_SHAPE;
  const size_t need = attn_fwd_naive_workspace_bytes(B, H, N);
  if (need == 0 || need > static_cast<size_t>(ATTN_NOALLOC_SCRATCH_BYTES))
    return ATTN_ERR_WORKSPACE;
  if ((st = check_device()) != ATTN_OK) return st;
  void* scratch = attn::noalloc_scratch_ptr();
  if (!scratch) return ATTN_ERR_CUDA;
  return attn::launch_naive(pack(q, k, v, o, lse, B, H, N, d, scale, causal), scratch,
                            reinterpret_cast<cudaStream_t>(stream));
}

namespace {

int validate_chain(const void* x, const void* b, const void* y, long long rows, int cols,
                   float alpha, int act) {
  if (!x || !b || !y) return ATTN_ERR_NULL;
  if (rows < 1 || cols < 1 || cols % 8 != 0) return ATTN_ERR_SHAPE;
  if (rows > (1ll << 62) / cols) return ATTN_ERR_SHAPE;
  if (!aligned(x, 16) || !aligned(b, 16) || !aligned(y, 16)) return ATTN_ERR_ALIGN;
  if (!std::isfinite(alpha)) return ATTN_ERR_SCALE;
  if (act < CHAIN_ACT_RELU || act > CHAIN_ACT_GELU_TANH) return ATTN_ERR_CAUSAL;
  return ATTN_OK;
}

}  // namespace

int chain_fused(const void* x, const void* b, void* y, long long rows, int cols, float alpha,
                int act, attn_stream_t stream) {
  int st = validate_chain(x, b, y, rows, cols, alpha, act);
  if (st != ATTN_OK) return st;
  if ((st = check_device()) != ATTN_OK) return st;
  return attn::launch_chain(x, b, y, nullptr, rows, cols, alpha, act, true,
                            reinterpret_cast<cudaStream_t>(stream));
}

int chain_unfused(const void* x, const void* b, void* y, void* tmp, long long rows, int cols,
                  float alpha, int act, attn_stream_t stream) {
  int st = validate_chain(x, b, y, rows, cols, alpha, act);
  if (st != ATTN_OK) return st;
  if (!tmp) return ATTN_ERR_NULL;
  if (!aligned(tmp, 16)) return ATTN_ERR_ALIGN;
  if ((st = check_device()) != ATTN_OK) return st;
  return attn::launch_chain(x, b, y, tmp, rows, cols, alpha, act, false,
                            reinterpret_cast<cudaStream_t>(stream));
}

int attn_last_device_error(attn_stream_t stream) {
  return attn::read_and_clear_device_error(reinterpret_cast<cudaStream_t>(stream));
}

int attn_set_wait_limit_ms(int ms) {
  if (ms < 1 || ms > 600000) return ATTN_ERR_SHAPE;
  attn::set_wait_limit_ms(ms);
  return ATTN_OK;
}

int attn_wait_limit_ms(void) { return attn::wait_limit_ms(); }

int attn_selftest_wait_timeout(int limit_ms, attn_stream_t stream) {
  if (limit_ms < 1 || limit_ms > 5000) return ATTN_ERR_SHAPE;
  int st = check_device();
  if (st != ATTN_OK) return st;
  return attn::launch_wait_timeout_selftest(limit_ms, reinterpret_cast<cudaStream_t>(stream));
}

int attn_selftest_exp2(const float* x, float* y, int n, attn_stream_t stream) {
  if (!x || !y) return ATTN_ERR_NULL;
  if (n < 1) return ATTN_ERR_SHAPE;
  if (!aligned(x, 4) || !aligned(y, 4)) return ATTN_ERR_ALIGN;
  int st = check_device();
  if (st != ATTN_OK) return st;
  return attn::launch_exp2_poly_selftest(x, y, n, reinterpret_cast<cudaStream_t>(stream));
}

const char* attn_status_string(int status) {
  switch (status) {
    case ATTN_OK: return "ATTN_OK";
    case ATTN_ERR_NULL: return "ATTN_ERR_NULL: a required pointer is NULL";
    case ATTN_ERR_SHAPE: return "ATTN_ERR_SHAPE: B, H or N out of range";
    case ATTN_ERR_HEADDIM: return "ATTN_ERR_HEADDIM: d must be 64 or 128";
    case ATTN_ERR_ALIGN: return "ATTN_ERR_ALIGN: pointer misaligned";
    case ATTN_ERR_SCALE: return "ATTN_ERR_SCALE: scale must be finite (FP8 descales finite and > 0)";
    case ATTN_ERR_CAUSAL: return "ATTN_ERR_CAUSAL: causal must be 0 or 1";
    case ATTN_ERR_WORKSPACE: return "ATTN_ERR_WORKSPACE: workspace too small";
    case ATTN_ERR_LAUNCH: return "ATTN_ERR_LAUNCH: kernel launch failed";
    case ATTN_ERR_UNSUPPORTED_DEVICE: return "ATTN_ERR_UNSUPPORTED_DEVICE: needs an sm_100 GPU";
    case ATTN_ERR_TIMEOUT: return "ATTN_ERR_TIMEOUT: a device-side bounded wait ran out";
    case ATTN_ERR_CUDA: return "ATTN_ERR_CUDA: a CUDA runtime call failed";
    case ATTN_ERR_WINDOW: return "ATTN_ERR_WINDOW: a window bound is below -1";
    default: return "unknown attn status";
  }
}

}  // extern "C"
