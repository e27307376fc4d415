// fused_fwd.cu - fused exact-attention forward for sm_100a (B200).
//
// What it computes: O = softmax(Q K^T * scale [+ causal mask]) V and the
// per-row log-sum-exp, for [B, H, N, d] bf16 tensors (the standard attention
// of the grasp.study lesson "The Computational Steps of Standard
// Self-Attention"), as one kernel that keeps the N x N scores and
// probabilities on chip and writes only O and lse (pratikdhanave.com, "The
// Attention Bottleneck - and How FlashAttention Fixed It", section "The fix:
// tiling and fusion, never touch HBM": tiles plus a running softmax
// normalisation, one kernel, HBM paid once).
//
// Work unit: one (batch*head, block of 256 query rows) per CTA, split into two
// 128-row query tiles "a" and "b" that ping-pong: while the softmax warps of
// one tile turn S into P, the tensor core runs the other tile's MMAs.
//
// Roles (320 threads):
//   warps 0-3  softmax + epilogue of query tile a (thread t owns row t)
//   warps 4-7  softmax + epilogue of query tile b
//   warp  8    TMA producer: Q tiles once, then K_0, V_0, K_1, V_1, ... into
//              a ring of shared-memory stages (128B-swizzled, mbarrier-tracked)
//   warp  9    tensor-memory allocator and single-thread tcgen05 MMA issuer
//
// Tensor memory (512 columns x 128 lanes, fp32): S_a [0,128), S_b [128,256),
// O_a [256, 256+d), O_b [256+d, 256+2d). P (bf16, two per column) overwrites
// the first 64 columns of its tile's S once S has been read into registers,
// and is the A operand of the P.V MMA straight from tensor memory.
//
// Online softmax (per row, in the log2 domain, x = s * scale * log2(e)):
//   m_tile = max over the tile, and the running maximum m is only raised when
//   m_tile > m + 8; then alpha = 2^(m_old - m_new) rescales l and the O row.
//   p = 2^(x - m) (at most 2^8 while m lags), l += sum p, O += P V.
//   At the end o = O / l and lse = (m + log2 l) * ln 2. Because the same m is
//   used for p, l and O, the result is the exact softmax whatever m is.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <mutex>

#include "../../include/attn.h"
#include "internal.h"
#include "sm100.cuh"
#include "tmem_io.cuh"
#include "watchdog.cuh"

namespace attn {

// Device-global error word (one per device that loads the library).
__device__ unsigned int g_device_error;

namespace {

constexpr int kTileRows = 128;           // query rows per tile == keys per KV tile
constexpr int kBlockRows = 256;          // query rows per CTA (two tiles)
constexpr int kThreads = 384;  // three warpgroups
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;     // warps 10 and 11 only give their registers away
// Registers per thread: what ptxas allocates at launch for 384 threads (the
// host refuses to launch otherwise), and the split after setmaxnreg. The
// split uses exactly the launch total.
constexpr int kRegsAtLaunch = 168;
constexpr int kRegsSoftmax = 224;
constexpr int kRegsOther = 56;
static_assert(128 * (2 * kRegsSoftmax + kRegsOther) == kThreads * kRegsAtLaunch,
              "register split must equal the launch allocation");
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: p <= 256 while m lags
constexpr uint64_t kWaitLimitNs = 2000000000ull;

// Which of a row's 64 (even, odd) column pairs take the FMA-pipe exponential
// (exp2_poly_pair) instead of the MUFU one; kPolyPeriod = 0 means none.
constexpr int kPolyPeriod = 4;
__host__ __device__ constexpr bool poly_pair(int cc) {
  return kPolyPeriod > 0 && cc % (kPolyPeriod > 0 ? kPolyPeriod : 1) == kPolyPeriod - 1;
}

template <int D>
struct Cfg {
  static constexpr int kTileBytes = kTileRows * D * 2;  // one 128 x D bf16 tile
  static constexpr int kAtoms = D / 64;                 // 128-byte swizzle atoms per row
  static constexpr int kAtomBytes = kTileRows * 128;    // 16 KiB
  static constexpr int kStages = (D == 128) ? 4 : 8;  // tile slots of the ring
  static constexpr int kUnits = kStages / 2;           // (V, K) units in flight
  static constexpr int kQOff = 0;
  static constexpr int kRingOff = 2 * kTileBytes;
  static constexpr int kBarOff = kRingOff + kStages * kTileBytes;
  // q_full, kv_full[S], kv_empty[S], s_full[2], p_ready[2], o_final[2], mma_done
  static constexpr int kNumBars = 1 + 2 * kStages + 6 + 1;
  static constexpr int kMiscOff = kBarOff + 8 * kNumBars;  // tmem base, abort flag
  static constexpr int kSmemBytes = kMiscOff + 16 + 1024;   // + alignment slack
  __host__ __device__ static constexpr uint32_t col_s(int g) { return g == 0 ? 0u : 128u; }
  __host__ __device__ static constexpr uint32_t col_o(int g) { return 256u + (g == 0 ? 0u : uint32_t(D)); }
};

struct FwdParams {
  void* o;
  float* lse;
  unsigned int* err;
  int N, BH, nqb, T;
  float scale_log2;
  int causal;
  uint64_t wait_limit_ns;
};

template <int D>
__device__ __forceinline__ void softmax_role(const FwdParams& p, uint32_t tmem, uint32_t bars,
                                             int bh, int q0, int n_kv, int g,
                                             const Watchdog& wd) {
  using C = Cfg<D>;
  const int warp = threadIdx.x / 32;
  const int tid = threadIdx.x % 128;
  const uint32_t lane_base = static_cast<uint32_t>(32 * (warp % 4)) << 16;
  const uint32_t tS = tmem + lane_base + C::col_s(g);
  const uint32_t tO = tmem + lane_base + C::col_o(g);
  const uint32_t bar_s_full = bars + 8u * (1 + 2 * C::kStages + g);
  const uint32_t bar_p_ready = bars + 8u * (1 + 2 * C::kStages + 2 + g);
  const uint32_t bar_o_final = bars + 8u * (1 + 2 * C::kStages + 4 + g);
  const int row_start = q0 + kTileRows * g;
  const int row = row_start + tid;
  const float c = p.scale_log2;

  float m_run = -INFINITY;
  float l_run = 0.0f;
  bool ok = true;
  for (int j = 0; j < n_kv; ++j) {
    if (!(ok = warp_wait(bar_s_full, j & 1, wd))) break;
    tc_fence_after_sync();
    uint32_t sr[128];
    tmem_ld_x128_wait(tS, sr);

    const int col0 = j * kTileRows;
    const bool need_mask = (p.causal && col0 + kTileRows - 1 > row_start) || (col0 + kTileRows > p.N);
    if (need_mask) {
      int lim = p.N - 1 - col0;
      if (p.causal) lim = min(lim, row - col0);
#pragma unroll
      for (int cc = 0; cc < 128; ++cc)
        if (cc > lim) sr[cc] = 0xff800000u;  // -inf
    }

    float mx[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) mx[u] = __uint_as_float(sr[u]);
#pragma unroll
    for (int cc = 8; cc < 128; cc += 2)
      mx[(cc / 2) % 8] = fmax3(mx[(cc / 2) % 8], __uint_as_float(sr[cc]), __uint_as_float(sr[cc + 1]));
    const float rmax = fmax3(fmax3(mx[0], mx[1], mx[2]), fmax3(mx[3], mx[4], mx[5]),
                             fmaxf(mx[6], mx[7]));
    const float m_tile = rmax * c;
    const bool raise = m_tile > m_run + kRescaleThreshold;
    const float m_new = raise ? m_tile : m_run;
    const float alpha = raise ? ex2_approx(m_run - m_new) : 1.0f;
    l_run *= alpha;
    if (j > 0 && __any_sync(0xffffffffu, raise)) {
      // O row *= alpha (threads that did not raise use alpha = 1)
#pragma unroll
      for (int ch = 0; ch < D / 32; ++ch) {
        uint32_t orr[32];
        tmem_ld_x32_wait(tO + ch * 32, orr);
#pragma unroll
        for (int u = 0; u < 32; ++u) orr[u] = __float_as_uint(__uint_as_float(orr[u]) * alpha);
        tmem_st_x32(tO + ch * 32, orr);
      }
    }
    m_run = m_new;
    const float neg_m = (m_run == -INFINITY) ? 0.0f : -m_run;

    // p = 2^(s * c - m) for the 64 (even, odd) column pairs: scaling and
    // summing in packed f32x2 form; most exponentials on the MUFU (ex2), the
    // pairs poly_pair picks on the FMA pipe (exp2_poly_pair).
    const uint64_t c2 = f2_pack(c, c);
    const uint64_t nm2 = f2_pack(neg_m, neg_m);
    uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
    uint32_t pk[64];
#pragma unroll
    for (int cc = 0; cc < 64; ++cc) {
      float x0, x1, p0, p1;
      f2_unpack(f2_fma(f2_pack(__uint_as_float(sr[2 * cc]), __uint_as_float(sr[2 * cc + 1])), c2, nm2),
                x0, x1);
      if (poly_pair(cc)) {
        exp2_poly_pair(x0, x1, p0, p1);
      } else {
        p0 = ex2_approx(x0);
        p1 = ex2_approx(x1);
      }
      acc[cc % 4] = f2_add(acc[cc % 4], f2_pack(p0, p1));
      pk[cc] = pack_bf16x2(p0, p1);
    }
    {
      float lo, hi;
      f2_unpack(f2_add(f2_add(acc[0], acc[1]), f2_add(acc[2], acc[3])), lo, hi);
      l_run += lo + hi;
    }
    tmem_st_x64(tS, pk);
    tmem_st_wait();
    tc_fence_before_sync();
    mbar_arrive(bar_p_ready);
  }
  if (ok) ok = warp_wait(bar_o_final, 0, wd);
  if (!ok) return;
  tc_fence_after_sync();

  // Epilogue: O / l -> bf16, lse in natural log.
  const float inv_l = 1.0f / l_run;
  const bool valid = row < p.N;
  uint4* orow = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.o) +
                                         (static_cast<size_t>(bh) * p.N + row) * D);
#pragma unroll
  for (int ch = 0; ch < D / 32; ++ch) {
    uint32_t orr[32];
    tmem_ld_x32_wait(tO + ch * 32, orr);
    uint32_t w[16];
#pragma unroll
    for (int u = 0; u < 16; ++u)
      w[u] = pack_bf16x2(__uint_as_float(orr[2 * u]) * inv_l, __uint_as_float(orr[2 * u + 1]) * inv_l);
    if (valid) {
#pragma unroll
      for (int u = 0; u < 4; ++u)
        orow[ch * 4 + u] = make_uint4(w[4 * u], w[4 * u + 1], w[4 * u + 2], w[4 * u + 3]);
    }
  }
  if (valid) {
    const float m_fin = (m_run == -INFINITY) ? 0.0f : m_run;
    p.lse[static_cast<size_t>(bh) * p.N + row] = (m_fin + __log2f(l_run)) * 0.69314718055994531f;
  }
}

template <int D>
__device__ __forceinline__ void producer_role(const CUtensorMap* tq, const CUtensorMap* tk,
                                              const CUtensorMap* tv, uint32_t base, uint32_t bars,
                                              int bh, int q0, int n_kv_b, const Watchdog& wd) {
  using C = Cfg<D>;
  const uint32_t sQ = base + C::kQOff;
  const uint32_t sRing = base + C::kRingOff;
  const uint32_t bar_q = bars;
  const uint64_t pol_q = l2_policy_evict_first();
  const uint64_t pol_kv = l2_policy_evict_last();

  mbar_arrive_expect_tx(bar_q, 2 * C::kTileBytes);
#pragma unroll
  for (int g = 0; g < 2; ++g)
#pragma unroll
    for (int a = 0; a < C::kAtoms; ++a)
      tma_load_3d_hint(sQ + g * C::kTileBytes + a * C::kAtomBytes, tq, bar_q, a * 64,
                       q0 + g * kTileRows, bh, pol_q);

  // K/V arrive in units that the MMA warp consumes together: unit 0 = K_0,
  // unit u >= 1 = (V_{u-1}, K_u), the last unit V only. A unit occupies two
  // tile slots of the ring (V in the first, K in the second) and has one full
  // and one empty barrier, so the MMA warp waits once per step for its tiles.
  const int n_units = n_kv_b + 1;
  int u = 0;
  for (; u < n_units; ++u) {
    const int us = u % C::kUnits;
    const uint32_t ph = (u / C::kUnits) & 1;
    const uint32_t bar_full = bars + 8u * (1 + us);
    const uint32_t bar_empty = bars + 8u * (1 + C::kStages + us);
    if (!wait_one(bar_empty, ph ^ 1u, wd)) break;
    const bool has_v = u >= 1;
    const bool has_k = u < n_kv_b;
    mbar_arrive_expect_tx(bar_full, (int(has_v) + int(has_k)) * C::kTileBytes);
    if (has_v) {
#pragma unroll
      for (int a = 0; a < C::kAtoms; ++a)
        tma_load_3d_hint(sRing + (2 * us) * C::kTileBytes + a * C::kAtomBytes, tv, bar_full,
                         a * 64, (u - 1) * kTileRows, bh, pol_kv);
    }
    if (has_k) {
#pragma unroll
      for (int a = 0; a < C::kAtoms; ++a)
        tma_load_3d_hint(sRing + (2 * us + 1) * C::kTileBytes + a * C::kAtomBytes, tk, bar_full,
                         a * 64, u * kTileRows, bh, pol_kv);
    }
  }
  // Teardown: every copy this thread issued must have landed before exit.
  drain_wait(bar_q, 0, wd);
  for (int w = (u > C::kUnits ? u - C::kUnits : 0); w < u; ++w)
    drain_wait(bars + 8u * (1 + w % C::kUnits), (w / C::kUnits) & 1, wd);
}

template <int D>
__device__ __forceinline__ void mma_role(uint32_t tmem, uint32_t base, uint32_t bars, int na,
                                         int nb, const Watchdog& wd) {
  using C = Cfg<D>;
  const uint32_t sQ = base + C::kQOff;
  const uint32_t sRing = base + C::kRingOff;
  const uint32_t bar_q = bars;
  const uint32_t bar_s_full0 = bars + 8u * (1 + 2 * C::kStages);
  const uint32_t bar_p_ready0 = bar_s_full0 + 16u;
  const uint32_t bar_o_final0 = bar_s_full0 + 32u;
  const uint32_t bar_mma_done = bar_s_full0 + 48u;
  constexpr uint32_t idesc_qk = idesc_bf16_f32(128, 128, 0, 0);
  constexpr uint32_t idesc_pv = idesc_bf16_f32(128, D, 0, 1);

  // unit u (see producer_role): V_{u-1} in tile slot 2 (u % kUnits), K_u in the next one
  auto par_of = [](int u) { return static_cast<uint32_t>((u / C::kUnits) & 1); };
  auto full_bar = [&](int u) { return bars + 8u * (1 + u % C::kUnits); };
  auto empty_bar = [&](int u) { return bars + 8u * (1 + C::kStages + u % C::kUnits); };
  auto v_slot = [](int u) { return 2 * (u % C::kUnits); };
  auto k_slot = [](int u) { return 2 * (u % C::kUnits) + 1; };

  // S_g = Q_g K^T : A = Q tile (K-major), B = K tile (K-major), 16-deep steps.
  auto issue_qk = [&](int g, int slot) {
    const uint32_t a0 = sQ + g * C::kTileBytes;
    const uint32_t b0 = sRing + slot * C::kTileBytes;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const uint32_t off = (kk >> 2) * C::kAtomBytes + (kk & 3) * 32;
      mma_ss(tmem + C::col_s(g), sdesc_sw128(a0 + off, 16, 1024), sdesc_sw128(b0 + off, 16, 1024),
             idesc_qk, kk > 0 ? 1u : 0u);
    }
  };
  // O_g += P_g V : A = P in tensor memory, B = V tile (MN-major), 16 keys per step.
  auto issue_pv = [&](int g, int slot, bool accumulate) {
    const uint32_t b0 = sRing + slot * C::kTileBytes;
#pragma unroll
    for (int kk = 0; kk < kTileRows / 16; ++kk)
      mma_ts(tmem + C::col_o(g), tmem + C::col_s(g) + kk * 8,
             sdesc_sw128(b0 + kk * 2048, C::kAtomBytes, 1024), idesc_pv,
             (accumulate || kk > 0) ? 1u : 0u);
  };

  bool ok = wait_one(bar_q, 0, wd) && wait_one(full_bar(0), par_of(0), wd);
  if (ok) {
    tc_fence_after_sync();
    issue_qk(0, k_slot(0));
    mma_commit(bar_s_full0);
    issue_qk(1, k_slot(0));
    mma_commit(bar_s_full0 + 8u);
    mma_commit(empty_bar(0));
  }
  for (int j = 0; ok && j < nb; ++j) {
    const int u = j + 1;  // V_j and K_{j+1}
    if (!(ok = wait_one(full_bar(u), par_of(u), wd))) break;
    if (j < na) {
      if (!(ok = wait_one(bar_p_ready0, j & 1, wd))) break;
      tc_fence_after_sync();
      issue_pv(0, v_slot(u), j > 0);
      if (j + 1 < na) {
        issue_qk(0, k_slot(u));
        mma_commit(bar_s_full0);
      } else {
        mma_commit(bar_o_final0);
      }
    }
    if (!(ok = wait_one(bar_p_ready0 + 8u, j & 1, wd))) break;
    tc_fence_after_sync();
    issue_pv(1, v_slot(u), j > 0);
    if (j + 1 < nb) {
      issue_qk(1, k_slot(u));
      mma_commit(bar_s_full0 + 8u);
    } else {
      mma_commit(bar_o_final0 + 8u);
    }
    mma_commit(empty_bar(u));
  }
  // Teardown: all MMAs this thread issued must be complete before the tensor
  // memory is freed.
  mma_commit(bar_mma_done);
  drain_wait(bar_mma_done, 0, wd);
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    fused_attn_fwd_kernel(const __grid_constant__ CUtensorMap tmap_q,
                          const __grid_constant__ CUtensorMap tmap_k,
                          const __grid_constant__ CUtensorMap tmap_v, const FwdParams p) {
  using C = Cfg<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;  // 128B swizzle wants 1024-byte alignment
  uint8_t* smem = smem_raw + (base - raw);
  const uint32_t bars = base + C::kBarOff;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kMiscOff);
  volatile uint32_t* abort_flag = tmem_slot + 1;

  const int warp = threadIdx.x / 32;
  const uint32_t lane = threadIdx.x % 32;

  // Work unit: heads are the slow index so co-resident CTAs share K/V in L2;
  // with causal masking the heaviest query blocks go first.
  const int bh = blockIdx.x / p.nqb;
  const int r = blockIdx.x % p.nqb;
  const int qblk = p.causal ? (p.nqb - 1 - r) : r;
  const int q0 = qblk * kBlockRows;
  const int na = p.causal ? min(p.T, q0 / kTileRows + 1) : p.T;
  const int nb = p.causal ? min(p.T, q0 / kTileRows + 2) : p.T;

  if (threadIdx.x == 0) {
    mbar_init(bars, 1);
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(bars + 8u * (1 + s), 1);
      mbar_init(bars + 8u * (1 + C::kStages + s), 1);
    }
    const uint32_t b6 = bars + 8u * (1 + 2 * C::kStages);
    mbar_init(b6 + 0, 1);    // s_full a
    mbar_init(b6 + 8, 1);    // s_full b
    mbar_init(b6 + 16, 128); // p_ready a
    mbar_init(b6 + 24, 128); // p_ready b
    mbar_init(b6 + 32, 1);   // o_final a
    mbar_init(b6 + 40, 1);   // o_final b
    mbar_init(b6 + 48, 1);   // mma_done
    *abort_flag = 0u;
    mbar_fence_init();
  }
  if (warp == kProducerWarp && lane == 0) {
    tma_prefetch_desc(&tmap_q);
    tma_prefetch_desc(&tmap_k);
    tma_prefetch_desc(&tmap_v);
  }
  if (warp == kMmaWarp) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(tmem_slot);
  const Watchdog wd{abort_flag, p.err, p.wait_limit_ns};

  if (warp < 8) {
    regs_increase<kRegsSoftmax>();
    const int g = warp / 4;
    softmax_role<D>(p, tmem, bars, bh, q0, g == 0 ? na : nb, g, wd);
  } else {
    regs_decrease<kRegsOther>();
    if (warp == kProducerWarp) {
      if (lane == 0) producer_role<D>(&tmap_q, &tmap_k, &tmap_v, base, bars, bh, q0, nb, wd);
    } else if (warp == kMmaWarp) {
      if (lane == 0) mma_role<D>(tmem, base, bars, na, nb, wd);
    }
  }
  __syncwarp();
  tc_fence_before_sync();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// Watchdog self-test: one warp waits on a barrier that nothing arrives on.
__global__ void wait_timeout_selftest_kernel(unsigned int* err, uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ uint32_t abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    abort_flag = 0u;
    mbar_fence_init();
  }
  __syncthreads();
  const Watchdog wd{&abort_flag, err, limit_ns};
  warp_wait(smem_u32(&bar), 0, wd);
  __syncwarp();
}

// ------------------------------------------------------------------- host

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult qres{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &qres) ==
            cudaSuccess &&
        qres == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

// [B*H, N, d] bf16 viewed as a 3-D tensor (d innermost); box = 64 columns
// (128 bytes, one swizzle atom) x 128 rows x 1 head; rows past N read as 0.
bool encode_qkv_map(CUtensorMap* m, const void* ptr, int BH, int N, int d) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N),
                        static_cast<cuuint64_t>(BH)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2,
                           static_cast<cuuint64_t>(N) * static_cast<cuuint64_t>(d) * 2};
  cuuint32_t box[3] = {64, static_cast<cuuint32_t>(kTileRows), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

unsigned int* device_error_word() {
  static unsigned int* ptrs[64] = {nullptr};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!ptrs[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_error) != cudaSuccess) return nullptr;
    ptrs[dev] = static_cast<unsigned int*>(p);
  }
  return ptrs[dev];
}

template <int D>
int launch_fused_d(const AttnArgs& a, cudaStream_t stream) {
  using C = Cfg<D>;
  const int BH = a.B * a.H;
  CUtensorMap mq, mk, mv;
  if (!encode_qkv_map(&mq, a.q, BH, a.N, D) || !encode_qkv_map(&mk, a.k, BH, a.N, D) ||
      !encode_qkv_map(&mv, a.v, BH, a.N, D))
    return ATTN_ERR_CUDA;
  unsigned int* err = device_error_word();
  if (!err) return ATTN_ERR_CUDA;
  FwdParams p{};
  p.o = a.o;
  p.lse = a.lse;
  p.err = err;
  p.N = a.N;
  p.BH = BH;
  p.nqb = (a.N + kBlockRows - 1) / kBlockRows;
  p.T = (a.N + kTileRows - 1) / kTileRows;
  p.scale_log2 = static_cast<float>(static_cast<double>(a.scale) * 1.4426950408889634);
  p.causal = a.causal;
  p.wait_limit_ns = kWaitLimitNs;
  const long long grid = static_cast<long long>(p.nqb) * BH;
  if (grid > 0x7fffffffLL) return ATTN_ERR_SHAPE;
  if (cudaFuncSetAttribute(fused_attn_fwd_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           C::kSmemBytes) != cudaSuccess)
    return ATTN_ERR_CUDA;
  // The register split inside the kernel assumes this exact allocation.
  cudaFuncAttributes fa{};
  if (cudaFuncGetAttributes(&fa, fused_attn_fwd_kernel<D>) != cudaSuccess) return ATTN_ERR_CUDA;
  if (fa.numRegs != kRegsAtLaunch || fa.maxThreadsPerBlock < kThreads) return ATTN_ERR_LAUNCH;
  fused_attn_fwd_kernel<D><<<static_cast<unsigned>(grid), kThreads, C::kSmemBytes, stream>>>(
      mq, mk, mv, p);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_LAUNCH;
}

}  // namespace

int launch_fused(const AttnArgs& a, cudaStream_t stream) {
  return a.d == 128 ? launch_fused_d<128>(a, stream) : launch_fused_d<64>(a, stream);
}

int read_and_clear_device_error(cudaStream_t stream) {
  unsigned int* err = device_error_word();
  if (!err) return ATTN_ERR_CUDA;
  unsigned int h = 0;
  if (cudaMemcpyAsync(&h, err, sizeof h, cudaMemcpyDeviceToHost, stream) != cudaSuccess)
    return ATTN_ERR_CUDA;
  if (cudaMemsetAsync(err, 0, sizeof h, stream) != cudaSuccess) return ATTN_ERR_CUDA;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return ATTN_ERR_CUDA;
  return (h & kDevErrTimeout) ? ATTN_ERR_TIMEOUT : ATTN_OK;
}

int launch_wait_timeout_selftest(int limit_ms, cudaStream_t stream) {
  unsigned int* err = device_error_word();
  if (!err) return ATTN_ERR_CUDA;
  wait_timeout_selftest_kernel<<<1, 32, 0, stream>>>(err,
                                                     static_cast<uint64_t>(limit_ms) * 1000000ull);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_LAUNCH;
}

}  // namespace attn
