// naive.cu - the deliberately unfused standard attention path.
//
// Three kernels, each reading its input from HBM and writing its output back,
// as the anylearn.cc page "Attention Is Memory-Bound, and Nobody Noticed for
// Five Years" traces the textbook implementation:
//   1. scores:  S = scale * Q K^T (bf16, causally masked entries = -inf)  -> HBM
//   2. softmax: P = softmax(S) row by row (fp32 math, bf16 out), lse (fp32) -> HBM
//   3. values:  O = P V (fp32 accumulate, bf16 out)                       -> HBM
// The N x N matrices S and P each cross the HBM boundary twice. This path is
// a measuring stick for that traffic, not a product path: its two matrix
// products run on the tensor cores (tcgen05 with TMA-fed tiles when N % 8 ==
// 0, warp-level mma.sync otherwise) so that it is bound by memory, as the
// pages say it is, rather than by arithmetic.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "../../include/attn.h"
#include "ctx_cache.h"
#include "internal.h"
#include "sm100.cuh"
#include "tmem_io.cuh"
#include "watchdog.cuh"

namespace attn {
namespace {

constexpr int kT = 128;          // output tile rows/cols
constexpr int kChunk = 64;       // keys per step of the P.V kernel
constexpr uint16_t kBf16NegInf = 0xFF80u;

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x2(uint32_t addr, uint32_t (&r)[2]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0, %1}, [%2];"
               : "=r"(r[0]), "=r"(r[1])
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

// c += a * b for one m16n8k16 bf16 tile, fp32 accumulate.
__device__ __forceinline__ void mma16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t bf16x2_bits(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// Eight consecutive bf16 of a row with `valid` readable elements starting at
// `p`; vector load when allowed, else element by element with zero fill.
__device__ __forceinline__ uint4 load8(const uint16_t* p, int valid, bool vec_ok) {
  if (vec_ok && valid >= 8) return *reinterpret_cast<const uint4*>(p);
  uint16_t e[8];
#pragma unroll
  for (int u = 0; u < 8; ++u) e[u] = (u < valid) ? p[u] : uint16_t(0);
  return make_uint4(e[0] | (uint32_t(e[1]) << 16), e[2] | (uint32_t(e[3]) << 16),
                    e[4] | (uint32_t(e[5]) << 16), e[6] | (uint32_t(e[7]) << 16));
}

// ----------------------------------------------------------------- scores
// One 128 x 128 tile of S per CTA (8 warps as 2 x 4, each 64 x 32).
template <int D>
__global__ void __launch_bounds__(256) naive_scores_kernel(const uint16_t* __restrict__ q,
                                                           const uint16_t* __restrict__ k,
                                                           uint16_t* __restrict__ S, int N,
                                                           float scale, int causal) {
  constexpr int LD = D + 8;       // padded smem row (elements)
  constexpr int LDS = kT + 8;     // staging row
  extern __shared__ __align__(16) uint16_t sm[];
  uint16_t* Qs = sm;
  uint16_t* Ks = sm + kT * LD;
  const int c0 = blockIdx.x * kT, r0 = blockIdx.y * kT, bh = blockIdx.z;
  const size_t head = static_cast<size_t>(bh) * N;
  uint16_t* Sh = S + head * N;
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const bool vec_ok = (N % 8) == 0;

  if (causal && c0 > r0 + kT - 1) {  // tile entirely above the diagonal
    for (int e = tid; e < kT * kT; e += 256) {
      const int r = r0 + e / kT, c = c0 + e % kT;
      if (r < N && c < N) Sh[static_cast<size_t>(r) * N + c] = kBf16NegInf;
    }
    return;
  }

  for (int e = tid; e < kT * (D / 8); e += 256) {
    const int r = e / (D / 8), cv = (e % (D / 8)) * 8;
    const uint4 zero = make_uint4(0, 0, 0, 0);
    *reinterpret_cast<uint4*>(Qs + r * LD + cv) =
        (r0 + r < N) ? *reinterpret_cast<const uint4*>(q + (head + r0 + r) * D + cv) : zero;
    *reinterpret_cast<uint4*>(Ks + r * LD + cv) =
        (c0 + r < N) ? *reinterpret_cast<const uint4*>(k + (head + c0 + r) * D + cv) : zero;
  }
  __syncthreads();

  const int wm = warp / 4, wn = warp % 4;
  float acc[4][4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int u = 0; u < 4; ++u) acc[i][j][u] = 0.0f;

#pragma unroll
  for (int kk = 0; kk < D; kk += 16) {
    uint32_t a[4][4], b[4][2];
#pragma unroll
    for (int mi = 0; mi < 4; ++mi)
      ldsm_x4(smem_addr(Qs + (wm * 64 + mi * 16 + (lane % 16)) * LD + kk + (lane / 16) * 8), a[mi]);
#pragma unroll
    for (int ni = 0; ni < 4; ++ni)
      ldsm_x2(smem_addr(Ks + (wn * 32 + ni * 8 + (lane % 8)) * LD + kk + ((lane / 8) % 2) * 8),
              b[ni]);
#pragma unroll
    for (int mi = 0; mi < 4; ++mi)
#pragma unroll
      for (int ni = 0; ni < 4; ++ni) mma16816(acc[mi][ni], a[mi], b[ni][0], b[ni][1]);
  }
  __syncthreads();

  // scale, mask, round to bf16, stage the tile in shared memory
  uint16_t* St = sm;
  const float ninf = __uint_as_float(0xff800000u);
#pragma unroll
  for (int mi = 0; mi < 4; ++mi)
#pragma unroll
    for (int ni = 0; ni < 4; ++ni)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int r = wm * 64 + mi * 16 + lane / 4 + 8 * h;
        const int c = wn * 32 + ni * 8 + (lane % 4) * 2;
        float v0 = acc[mi][ni][2 * h] * scale, v1 = acc[mi][ni][2 * h + 1] * scale;
        if (causal) {
          if (c0 + c > r0 + r) v0 = ninf;
          if (c0 + c + 1 > r0 + r) v1 = ninf;
        }
        *reinterpret_cast<uint32_t*>(St + r * LDS + c) = bf16x2_bits(v0, v1);
      }
  __syncthreads();

  if (vec_ok && r0 + kT <= N && c0 + kT <= N) {
    for (int e = tid; e < kT * (kT / 8); e += 256) {
      const int r = e / (kT / 8), cv = (e % (kT / 8)) * 8;
      *reinterpret_cast<uint4*>(Sh + static_cast<size_t>(r0 + r) * N + c0 + cv) =
          *reinterpret_cast<const uint4*>(St + r * LDS + cv);
    }
  } else {
    for (int e = tid; e < kT * kT; e += 256) {
      const int r = e / kT, c = e % kT;
      if (r0 + r < N && c0 + c < N) Sh[static_cast<size_t>(r0 + r) * N + c0 + c] = St[r * LDS + c];
    }
  }
}

// ---------------------------------------------------------------- softmax
// One CTA per row of S; each thread keeps EPT elements of the row in registers
// so S is read once and P written once.
template <int EPT>
__global__ void __launch_bounds__(512) naive_softmax_kernel(const uint16_t* __restrict__ S, uint16_t* __restrict__ P,
                                     float* __restrict__ lse, int N) {
  __shared__ float red[32];
  const size_t row = blockIdx.x;
  const uint16_t* srow = S + row * N;
  uint16_t* prow = P + row * N;
  const int T = blockDim.x, tid = threadIdx.x, lane = tid % 32, warp = tid / 32;
  const int nwarps = T / 32;
  const bool vec = (N % 8) == 0;
  float x[EPT];
  const float ninf = __uint_as_float(0xff800000u);

  if (vec) {
#pragma unroll
    for (int i = 0; i < EPT / 8; ++i) {
      const int e = (tid + i * T) * 8;
      uint4 w = make_uint4(0xFF80FF80u, 0xFF80FF80u, 0xFF80FF80u, 0xFF80FF80u);
      if (e < N) w = *reinterpret_cast<const uint4*>(srow + e);
      const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        x[i * 8 + 2 * u] = __uint_as_float(ws[u] << 16);
        x[i * 8 + 2 * u + 1] = __uint_as_float(ws[u] & 0xffff0000u);
      }
    }
  } else {
#pragma unroll
    for (int i = 0; i < EPT; ++i) {
      const int e = tid + i * T;
      x[i] = (e < N) ? __uint_as_float(uint32_t(srow[e]) << 16) : ninf;
    }
  }

  float m = ninf;
#pragma unroll
  for (int i = 0; i < EPT; ++i) m = fmaxf(m, x[i]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if (lane == 0) red[warp] = m;
  __syncthreads();
  m = ninf;
  for (int w = 0; w < nwarps; ++w) m = fmaxf(m, red[w]);
  __syncthreads();

  const float l2e = 1.4426950408889634f;
  float s = 0.0f;
#pragma unroll
  for (int i = 0; i < EPT; ++i) {
    x[i] = exp2f((x[i] - m) * l2e);
    s += x[i];
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if (lane == 0) red[warp] = s;
  __syncthreads();
  s = 0.0f;
  for (int w = 0; w < nwarps; ++w) s += red[w];
  const float inv = 1.0f / s;

  if (vec) {
#pragma unroll
    for (int i = 0; i < EPT / 8; ++i) {
      const int e = (tid + i * T) * 8;
      if (e < N) {
        uint4 w;
        w.x = bf16x2_bits(x[i * 8 + 0] * inv, x[i * 8 + 1] * inv);
        w.y = bf16x2_bits(x[i * 8 + 2] * inv, x[i * 8 + 3] * inv);
        w.z = bf16x2_bits(x[i * 8 + 4] * inv, x[i * 8 + 5] * inv);
        w.w = bf16x2_bits(x[i * 8 + 6] * inv, x[i * 8 + 7] * inv);
        *reinterpret_cast<uint4*>(prow + e) = w;
      }
    }
  } else {
#pragma unroll
    for (int i = 0; i < EPT; ++i) {
      const int e = tid + i * T;
      if (e < N) {
        __nv_bfloat16 h = __float2bfloat16_rn(x[i] * inv);
        prow[e] = *reinterpret_cast<uint16_t*>(&h);
      }
    }
  }
  if (tid == 0) lse[row] = m + logf(s);
}

// ----------------------------------------------------------------- values
// O tile of 128 rows x D per CTA; 8 warps, each 16 rows x D; keys in chunks
// of 64 with the next chunk prefetched into registers during the MMAs.
template <int D>
__global__ void __launch_bounds__(256) naive_values_kernel(const uint16_t* __restrict__ P,
                                                           const uint16_t* __restrict__ V,
                                                           uint16_t* __restrict__ O, int N) {
  constexpr int LDP = kChunk + 8;
  constexpr int LDV = D + 8;
  constexpr int PV = kT * kChunk / 8 / 256;  // uint4 of P per thread per chunk (4)
  constexpr int VV = kChunk * D / 8 / 256;   // uint4 of V per thread per chunk (2 or 4)
  extern __shared__ __align__(16) uint16_t sm[];
  uint16_t* Ps = sm;
  uint16_t* Vs = sm + kT * LDP;
  const int r0 = blockIdx.x * kT, bh = blockIdx.y;
  const size_t head = static_cast<size_t>(bh) * N;
  const uint16_t* Ph = P + head * N;
  const uint16_t* Vh = V + head * D;
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const bool vec_ok = (N % 8) == 0;

  uint4 pr[PV], vr[VV];
  auto fetch = [&](int kv0) {
#pragma unroll
    for (int i = 0; i < PV; ++i) {
      const int e = tid + i * 256, r = e / (kChunk / 8), cv = (e % (kChunk / 8)) * 8;
      const int valid = (r0 + r < N) ? max(0, min(8, N - (kv0 + cv))) : 0;
      pr[i] = valid > 0 ? load8(Ph + static_cast<size_t>(r0 + r) * N + kv0 + cv, valid, vec_ok)
                        : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int i = 0; i < VV; ++i) {
      const int e = tid + i * 256, r = e / (D / 8), cv = (e % (D / 8)) * 8;
      vr[i] = (kv0 + r < N) ? *reinterpret_cast<const uint4*>(Vh + static_cast<size_t>(kv0 + r) * D + cv)
                            : make_uint4(0, 0, 0, 0);
    }
  };
  auto stash = [&]() {
#pragma unroll
    for (int i = 0; i < PV; ++i) {
      const int e = tid + i * 256, r = e / (kChunk / 8), cv = (e % (kChunk / 8)) * 8;
      *reinterpret_cast<uint4*>(Ps + r * LDP + cv) = pr[i];
    }
#pragma unroll
    for (int i = 0; i < VV; ++i) {
      const int e = tid + i * 256, r = e / (D / 8), cv = (e % (D / 8)) * 8;
      *reinterpret_cast<uint4*>(Vs + r * LDV + cv) = vr[i];
    }
  };

  float acc[D / 8][4];
#pragma unroll
  for (int n = 0; n < D / 8; ++n)
#pragma unroll
    for (int u = 0; u < 4; ++u) acc[n][u] = 0.0f;

  fetch(0);
  for (int kv0 = 0; kv0 < N; kv0 += kChunk) {
    stash();
    __syncthreads();
    if (kv0 + kChunk < N) fetch(kv0 + kChunk);
#pragma unroll
    for (int kk = 0; kk < kChunk; kk += 16) {
      uint32_t a[4];
      ldsm_x4(smem_addr(Ps + (warp * 16 + (lane % 16)) * LDP + kk + (lane / 16) * 8), a);
#pragma unroll
      for (int nb = 0; nb < D / 16; ++nb) {
        uint32_t b[4];
        ldsm_x4_trans(smem_addr(Vs + (kk + (lane % 16)) * LDV + nb * 16 + (lane / 16) * 8), b);
        mma16816(acc[2 * nb], a, b[0], b[1]);
        mma16816(acc[2 * nb + 1], a, b[2], b[3]);
      }
    }
    __syncthreads();
  }

#pragma unroll
  for (int n = 0; n < D / 8; ++n)
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int r = r0 + warp * 16 + lane / 4 + 8 * h;
      const int c = n * 8 + (lane % 4) * 2;
      if (r < N)
        *reinterpret_cast<uint32_t*>(O + (head + r) * D + c) =
            bf16x2_bits(acc[n][2 * h], acc[n][2 * h + 1]);
    }
}

// ------------------------------------------- tcgen05 kernels (N % 8 == 0)
// The same two matrix products on the 5th-generation tensor cores, with TMA
// moving every tile: S row blocks stream out of shared memory through TMA
// stores, P and V tiles stream in through TMA loads, so the products keep up
// with HBM and the path's time is the traffic it is there to show. (S and P
// are [B*H, N, N] bf16 arrays; a TMA row stride must be a multiple of 16
// bytes, hence N % 8 == 0; other N take the kernels above.)
//
// Roles (192 threads): warp 0 TMA producer, warp 1 tensor-memory allocator
// and MMA issuer, warps 2-5 epilogue (thread = tile row; warp w reaches
// tensor-memory lanes 32 (w % 4) .. + 31).
constexpr int kTcThreads = 192;

struct TcBars {
  // byte offsets of the mbarriers from the barrier area
  __host__ __device__ static constexpr uint32_t full(int s) { return 8u * s; }  // s < 4
  __host__ __device__ static constexpr uint32_t empty(int s) { return 8u * (4 + s); }
  __host__ __device__ static constexpr uint32_t acc_full(int b) { return 8u * (8 + b); }  // b < 2
  __host__ __device__ static constexpr uint32_t acc_empty(int b) { return 8u * (10 + b); }
  static constexpr uint32_t kQFull = 8u * 12;
  static constexpr uint32_t kMmaDone = 8u * 13;
  static constexpr int kCount = 14;
};

// S = scale * Q K^T for 128 query rows of one head (all N keys), written to
// HBM as bf16 with causally masked entries -inf. The tensor core fills one of
// two S buffers in tensor memory while the epilogue drains the other into a
// swizzled staging tile that two TMA stores (64 columns each) copy out.
template <int D>
__global__ void __launch_bounds__(kTcThreads, 1)
    naive_scores_tc_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                           const __grid_constant__ CUtensorMap ts, int N, int nqb, float scale,
                           int causal, unsigned int* err, uint64_t wait_limit_ns) {
  constexpr int kTile = kT * D * 2;            // Q or K tile bytes
  constexpr int kAtom = kT * 128;              // 128 rows x 128 bytes
  constexpr int kStages = 3;
  constexpr int kStage = kT * kT * 2;          // staging tile, 32 KiB (two atoms)
  constexpr uint32_t kRingOff = kTile, kStageOff = kRingOff + kStages * kTile;
  constexpr uint32_t kBarOff = kStageOff + 2 * kStage;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t base = (smem_addr(smem_raw) + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - smem_addr(smem_raw));
  const uint32_t bars = base + kBarOff;
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + kBarOff + 8 * TcBars::kCount);
  volatile uint32_t* abort_flag = misc + 1;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int bh = blockIdx.x / nqb, r0 = (blockIdx.x % nqb) * kT;
  const int T = (N + kT - 1) / kT;
  // key tiles with at least one allowed key for some row of the block
  const int n_mma = causal ? min(T, r0 / kT + 1) : T;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 4; ++i) {
      mbar_init(bars + TcBars::full(i), 1);
      mbar_init(bars + TcBars::empty(i), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bars + TcBars::acc_full(b), 1);
      mbar_init(bars + TcBars::acc_empty(b), 128);
    }
    mbar_init(bars + TcBars::kQFull, 1);
    mbar_init(bars + TcBars::kMmaDone, 1);
    *abort_flag = 0u;
    mbar_fence_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_addr(misc), 256);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(misc);
  const Watchdog wd{abort_flag, err, wait_limit_ns};

  if (warp == 0) {
    if (lane == 0) {
      const uint64_t pol = l2_policy_evict_last();
      mbar_arrive_expect_tx(bars + TcBars::kQFull, kTile);
      for (int a = 0; a < D / 64; ++a)
        tma_load_3d_hint(base + a * kAtom, &tq, bars + TcBars::kQFull, a * 64, r0, bh, pol);
      int j = 0;
      for (; j < n_mma; ++j) {
        const int s = j % kStages;
        if (!wait_one(bars + TcBars::empty(s), ((j / kStages) & 1) ^ 1u, wd)) break;
        mbar_arrive_expect_tx(bars + TcBars::full(s), kTile);
        for (int a = 0; a < D / 64; ++a)
          tma_load_3d_hint(base + kRingOff + s * kTile + a * kAtom, &tk, bars + TcBars::full(s), a * 64,
                           j * kT, bh, pol);
      }
      drain_wait(bars + TcBars::kQFull, 0, wd);
      for (int w = (j > kStages ? j - kStages : 0); w < j; ++w)
        drain_wait(bars + TcBars::full(w % kStages), (w / kStages) & 1, wd);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, 128, 0, 0);
      bool ok = wait_one(bars + TcBars::kQFull, 0, wd);
      for (int j = 0; ok && j < n_mma; ++j) {
        const int s = j % kStages, b = j & 1;
        if (!(ok = wait_one(bars + TcBars::full(s), (j / kStages) & 1, wd))) break;
        if (!(ok = wait_one(bars + TcBars::acc_empty(b), ((j >> 1) & 1) ^ 1u, wd))) break;
        tc_fence_after_sync();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * kAtom + (kk & 3) * 32;
          mma_ss(tmem + 128u * b, sdesc_sw128(base + off, 16, 1024),
                 sdesc_sw128(base + kRingOff + s * kTile + off, 16, 1024), idesc, kk > 0 ? 1u : 0u);
        }
        mma_commit(bars + TcBars::acc_full(b));
        mma_commit(bars + TcBars::empty(s));
      }
      mma_commit(bars + TcBars::kMmaDone);
      drain_wait(bars + TcBars::kMmaDone, 0, wd);
    }
  } else {
    // epilogue: thread = row r of the block
    const int r = 32 * (warp % 4) + lane;
    const int row = r0 + r;
    const uint32_t lane_base = static_cast<uint32_t>(32 * (warp % 4)) << 16;
    const bool leader = threadIdx.x == 64;
    bool ok = true;
    for (int j = 0; j < T; ++j) {
      const int b = j & 1;
      const uint32_t stage = base + kStageOff + b * kStage;
      // the store that last read this staging tile (two tiles ago) has finished reading
      if (leader) bulk_wait_read<1>();
      named_barrier_sync(1, 128);
      const int col0 = j * kT;
      if (j < n_mma) {
        if (ok) ok = warp_wait(bars + TcBars::acc_full(b), (j >> 1) & 1, wd);
        tc_fence_after_sync();
        const int lim = causal ? row - col0 : kT;  // columns cc > lim are masked
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
          uint32_t v[32];
          if (ok) tmem_ld_x32_wait(tmem + lane_base + 128u * b + ch * 32, v);
          uint32_t w[16];
#pragma unroll
          for (int u = 0; u < 16; ++u) {
            const int c = ch * 32 + 2 * u;
            const float s0 = c > lim ? -INFINITY : __uint_as_float(v[2 * u]) * scale;
            const float s1 = c + 1 > lim ? -INFINITY : __uint_as_float(v[2 * u + 1]) * scale;
            w[u] = bf16x2_bits(s0, s1);
          }
          // 16-byte chunk q of this row's 64-column atom goes to chunk q ^ (r & 7)
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int chunk = (ch % 2) * 4 + q;
            uint8_t* dst = smem + (stage - base) + (ch / 2) * kAtom + r * 128 + ((chunk ^ (r & 7)) * 16);
            *reinterpret_cast<uint4*>(dst) = make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
          }
        }
        tc_fence_before_sync();
        mbar_arrive(bars + TcBars::acc_empty(b));
      } else {
        // every key of the tile is after every row of the block: all -inf
        const uint4 ninf = make_uint4(0xFF80FF80u, 0xFF80FF80u, 0xFF80FF80u, 0xFF80FF80u);
#pragma unroll
        for (int q = 0; q < 16; ++q)
          *reinterpret_cast<uint4*>(smem + (stage - base) + (q / 8) * kAtom + r * 128 + (q % 8) * 16) = ninf;
      }
      fence_proxy_async_smem();
      named_barrier_sync(1, 128);
      if (leader) {
        tma_store_3d(&ts, stage, col0, r0, bh);
        if (col0 + 64 < N) tma_store_3d(&ts, stage + kAtom, col0 + 64, r0, bh);
        bulk_commit();
      }
    }
    if (leader) bulk_wait_all();
  }
  __syncwarp();
  tc_fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, 256);
  }
}

// O = P V for 128 query rows of one head: P and V tiles of 128 keys stream
// through a ring (every P tile is read, as the unfused algorithm reads all of
// P; tiles wholly above the causal diagonal are all zero and skip the MMA).
template <int D>
__global__ void __launch_bounds__(kTcThreads, 1)
    naive_values_tc_kernel(const __grid_constant__ CUtensorMap tp, const __grid_constant__ CUtensorMap tv,
                           uint16_t* __restrict__ O, int N, int nqb, int causal, unsigned int* err,
                           uint64_t wait_limit_ns) {
  constexpr int kPTile = kT * kT * 2;          // 32 KiB
  constexpr int kVTile = kT * D * 2;
  constexpr int kAtom = kT * 128;
  constexpr int kUnit = kPTile + kVTile;
  constexpr int kStages = 3;
  constexpr uint32_t kBarOff = kStages * kUnit;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t base = (smem_addr(smem_raw) + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - smem_addr(smem_raw));
  const uint32_t bars = base + kBarOff;
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + kBarOff + 8 * TcBars::kCount);
  volatile uint32_t* abort_flag = misc + 1;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int bh = blockIdx.x / nqb, r0 = (blockIdx.x % nqb) * kT;
  const int T = (N + kT - 1) / kT;
  const int n_mma = causal ? min(T, r0 / kT + 1) : T;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 4; ++i) {
      mbar_init(bars + TcBars::full(i), 1);
      mbar_init(bars + TcBars::empty(i), 1);
    }
    mbar_init(bars + TcBars::acc_full(0), 1);
    mbar_init(bars + TcBars::kMmaDone, 1);
    *abort_flag = 0u;
    mbar_fence_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_addr(misc), 128);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(misc);
  const Watchdog wd{abort_flag, err, wait_limit_ns};

  if (warp == 0) {
    if (lane == 0) {
      const uint64_t pol_p = l2_policy_evict_first();
      const uint64_t pol_v = l2_policy_evict_last();
      int j = 0;
      for (; j < T; ++j) {
        const int s = j % kStages;
        if (!wait_one(bars + TcBars::empty(s), ((j / kStages) & 1) ^ 1u, wd)) break;
        const uint32_t unit = base + s * kUnit;
        mbar_arrive_expect_tx(bars + TcBars::full(s), kUnit);
        for (int a = 0; a < 2; ++a)
          tma_load_3d_hint(unit + a * kAtom, &tp, bars + TcBars::full(s), j * kT + a * 64, r0, bh, pol_p);
        for (int a = 0; a < D / 64; ++a)
          tma_load_3d_hint(unit + kPTile + a * kAtom, &tv, bars + TcBars::full(s), a * 64, j * kT, bh,
                           pol_v);
      }
      for (int w = (j > kStages ? j - kStages : 0); w < j; ++w)
        drain_wait(bars + TcBars::full(w % kStages), (w / kStages) & 1, wd);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, D, 0, 1);
      bool ok = true;
      for (int j = 0; ok && j < T; ++j) {
        const int s = j % kStages;
        if (!(ok = wait_one(bars + TcBars::full(s), (j / kStages) & 1, wd))) break;
        if (j < n_mma) {
          tc_fence_after_sync();
          const uint32_t unit = base + s * kUnit;
#pragma unroll
          for (int kk = 0; kk < kT / 16; ++kk) {
            // A = P tile (K-major: 128 rows, keys in two 128-byte atoms), B =
            // V tile (MN-major: one 128-byte row of d per key)
            const uint32_t a_off = (kk >> 2) * kAtom + (kk & 3) * 32;
            mma_ss(tmem, sdesc_sw128(unit + a_off, 16, 1024),
                   sdesc_sw128(unit + kPTile + kk * 2048, kAtom, 1024), idesc,
                   (j > 0 || kk > 0) ? 1u : 0u);
          }
        }
        mma_commit(bars + TcBars::empty(s));
      }
      mma_commit(bars + TcBars::acc_full(0));
      mma_commit(bars + TcBars::kMmaDone);
      drain_wait(bars + TcBars::kMmaDone, 0, wd);
    }
  } else {
    const int r = 32 * (warp % 4) + lane;
    const int row = r0 + r;
    const uint32_t lane_base = static_cast<uint32_t>(32 * (warp % 4)) << 16;
    if (warp_wait(bars + TcBars::acc_full(0), 0, wd)) {
      tc_fence_after_sync();
      uint16_t* orow = O + (static_cast<size_t>(bh) * N + row) * D;
#pragma unroll
      for (int ch = 0; ch < D / 32; ++ch) {
        uint32_t v[32];
        tmem_ld_x32_wait(tmem + lane_base + ch * 32, v);
        if (row < N) {
#pragma unroll
          for (int q = 0; q < 4; ++q)
            *reinterpret_cast<uint4*>(orow + ch * 32 + q * 8) = make_uint4(
                bf16x2_bits(__uint_as_float(v[8 * q]), __uint_as_float(v[8 * q + 1])),
                bf16x2_bits(__uint_as_float(v[8 * q + 2]), __uint_as_float(v[8 * q + 3])),
                bf16x2_bits(__uint_as_float(v[8 * q + 4]), __uint_as_float(v[8 * q + 5])),
                bf16x2_bits(__uint_as_float(v[8 * q + 6]), __uint_as_float(v[8 * q + 7])));
        }
      }
    }
  }
  __syncwarp();
  tc_fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, 128);
  }
}

template <int D>
int launch_naive_tc(const AttnArgs& a, uint16_t* S, uint16_t* P, float* lse, cudaStream_t stream,
                    int softmax_ept, int softmax_threads) {
  const int N = a.N, BH = a.B * a.H;
  const int nqb = (N + kT - 1) / kT;
  CUtensorMap mq, mk, ms, mp, mv;
  if (!encode_bf16_tiled_3d(&mq, a.q, D, N, BH, 64, kT) || !encode_bf16_tiled_3d(&mk, a.k, D, N, BH, 64, kT) ||
      !encode_bf16_tiled_3d(&ms, S, N, N, BH, 64, kT) || !encode_bf16_tiled_3d(&mp, P, N, N, BH, 64, kT) ||
      !encode_bf16_tiled_3d(&mv, a.v, D, N, BH, 64, kT))
    return ATTN_ERR_CUDA;
  unsigned int* err = library_error_word();
  if (!err) return ATTN_ERR_CUDA;
  const uint64_t limit = static_cast<uint64_t>(wait_limit_ms()) * 1000000ull;
  const long long grid = static_cast<long long>(nqb) * BH;
  if (grid > 0x7fffffffLL) return ATTN_ERR_SHAPE;
  static CtxCache<int> prep;
  int st = ATTN_ERR_CUDA;
  constexpr int kScoresSmem = kT * D * 2 * 4 + 2 * kT * kT * 2 + 8 * TcBars::kCount + 16 + 1024;
  constexpr int kValuesSmem = 3 * (kT * kT * 2 + kT * D * 2) + 8 * TcBars::kCount + 16 + 1024;
  static_assert(kScoresSmem <= 227 * 1024 && kValuesSmem <= 227 * 1024, "shared memory");
  if (!prep.get(&st, [](int* out) {
        *out = (cudaFuncSetAttribute(naive_scores_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     kScoresSmem) == cudaSuccess &&
                cudaFuncSetAttribute(naive_values_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     kValuesSmem) == cudaSuccess)
                   ? ATTN_OK
                   : ATTN_ERR_CUDA;
        return *out == ATTN_OK;
      }))
    return ATTN_ERR_CUDA;
  naive_scores_tc_kernel<D><<<static_cast<unsigned>(grid), kTcThreads, kScoresSmem, stream>>>(
      mq, mk, ms, N, nqb, a.scale, a.causal, err, limit);
  if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_LAUNCH;
  const unsigned rows = static_cast<unsigned>(static_cast<size_t>(BH) * N);
  switch (softmax_ept) {
    case 8: naive_softmax_kernel<8><<<rows, softmax_threads, 0, stream>>>(S, P, lse, N); break;
    case 16: naive_softmax_kernel<16><<<rows, softmax_threads, 0, stream>>>(S, P, lse, N); break;
    case 32: naive_softmax_kernel<32><<<rows, softmax_threads, 0, stream>>>(S, P, lse, N); break;
    default: naive_softmax_kernel<64><<<rows, softmax_threads, 0, stream>>>(S, P, lse, N); break;
  }
  if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_LAUNCH;
  naive_values_tc_kernel<D><<<static_cast<unsigned>(grid), kTcThreads, kValuesSmem, stream>>>(
      mp, mv, static_cast<uint16_t*>(a.o), N, nqb, a.causal, err, limit);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_LAUNCH;
}

template <int D>
int launch_naive_d(const AttnArgs& a, void* workspace, cudaStream_t stream) {
  const int N = a.N, BH = a.B * a.H;
  uint16_t* S = static_cast<uint16_t*>(workspace);
  uint16_t* P = S + static_cast<size_t>(BH) * N * N;
  const auto* q = static_cast<const uint16_t*>(a.q);
  const auto* k = static_cast<const uint16_t*>(a.k);
  const auto* v = static_cast<const uint16_t*>(a.v);
  auto* o = static_cast<uint16_t*>(a.o);
  const int tiles = (N + kT - 1) / kT;
  // softmax launch shape: EPT elements per thread, T threads per row
  int ept = 8;
  while (ept < 64 && (N + ept - 1) / ept > 256) ept *= 2;
  const int T = ((N + ept - 1) / ept + 31) / 32 * 32;
  if (T > 512) return ATTN_ERR_SHAPE;
  if (N % 8 == 0) return launch_naive_tc<D>(a, S, P, a.lse, stream, ept, T);
  if (BH > 65535) return ATTN_ERR_SHAPE;

  const int smem_scores = 2 * kT * (D + 8) * 2;
  if (cudaFuncSetAttribute(naive_scores_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           smem_scores) != cudaSuccess)
    return ATTN_ERR_CUDA;
  naive_scores_kernel<D><<<dim3(tiles, tiles, BH), 256, smem_scores, stream>>>(q, k, S, N, a.scale,
                                                                              a.causal);
  if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_LAUNCH;

  const unsigned rows = static_cast<unsigned>(static_cast<size_t>(BH) * N);
  switch (ept) {
    case 8: naive_softmax_kernel<8><<<rows, T, 0, stream>>>(S, P, a.lse, N); break;
    case 16: naive_softmax_kernel<16><<<rows, T, 0, stream>>>(S, P, a.lse, N); break;
    case 32: naive_softmax_kernel<32><<<rows, T, 0, stream>>>(S, P, a.lse, N); break;
    default: naive_softmax_kernel<64><<<rows, T, 0, stream>>>(S, P, a.lse, N); break;
  }
  if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_LAUNCH;

  const int smem_values = (kT * (kChunk + 8) + kChunk * (D + 8)) * 2;
  if (cudaFuncSetAttribute(naive_values_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           smem_values) != cudaSuccess)
    return ATTN_ERR_CUDA;
  naive_values_kernel<D><<<dim3(tiles, BH), 256, smem_values, stream>>>(P, v, o, N);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_LAUNCH;
}

}  // namespace

int launch_naive(const AttnArgs& a, void* workspace, cudaStream_t stream) {
  return a.d == 128 ? launch_naive_d<128>(a, workspace, stream)
                    : launch_naive_d<64>(a, workspace, stream);
}

// ------------------------------------------------- no-allocation variant
// Scratch for attn_fwd_naive_noalloc: S and P live here instead of in a
// caller-provided workspace. The array is part of the library image, so every
// GPU that loads the library reserves it until the process exits.
static __device__ __align__(256) unsigned char g_noalloc_scratch[ATTN_NOALLOC_SCRATCH_BYTES];

// Device address of g_noalloc_scratch on the current device. In host code the
// array's name is only a host-side stand-in, so the address is looked up with
// cudaGetSymbolAddress, with the device current, once per CUDA context (a
// context re-created after cudaDeviceReset gets a fresh lookup) and cached.
void* noalloc_scratch_ptr() {
  static CtxCache<void*> cache;
  void* ptr = nullptr;
  if (!cache.get(&ptr, [](void** out) {
        return cudaGetSymbolAddress(out, g_noalloc_scratch) == cudaSuccess;
      }))
    return nullptr;
  return ptr;
}

}  // namespace attn
