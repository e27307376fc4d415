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
// Work unit: one (batch*head, block of 256 query rows), split into two
// 128-row query tiles "a" and "b" that ping-pong: while the softmax warps of
// one tile turn S into P, the tensor core runs the other tile's MMAs. The
// square problem runs a persistent grid: one CTA per SM walks its work units
// (square_unit) on the same barriers and buffers, starting each unit's loads
// while the previous one finishes.
//
// Roles (384 threads):
//   warps 0-3  softmax + epilogue of query tile a (thread t owns row t)
//   warps 4-7  softmax + epilogue of query tile b
//   warp  8    TMA producer: Q tiles, then K_0, (V_0, K_1), (V_1, K_2), ...
//              into a ring of shared-memory stages (128B-swizzled,
//              mbarrier-tracked)
//   warp  9    tensor-memory allocator and single-thread tcgen05 MMA issuer
//   warps 10-11 only hand their registers to the softmax warps (setmaxnreg)
//
// The kv instantiation (kKV = true) serves Nq query rows against N keys with
// the keys of each head cut into ranges that separate CTAs attend to: a CTA is
// (head, key range, query block); with Nq <= 128 its one query tile is shared
// by both softmax warpgroups, which take alternate KV tiles and merge their
// (O, m, l) at the end. Several ranges leave fp32 partial (O, lse) pairs that
// lse_combine_kernel (combine.cu) merges. The same instantiation applies key
// windows around each query's position (tiles outside every window are not
// loaded) and an optional per-head linear distance bias.
//
// The FP8 instantiation (kF8 = true, square problem, d = 128) takes E4M3 Q,
// K, V, runs both products as tcgen05 kind::f8f6f4 MMAs and stores P as four
// E4M3 values per tensor-memory column (32 columns). The kBias instantiation
// of the square problem adds the per-head linear distance bias, and the kWin
// one applies key windows: each work unit starts at the KV tile of its first
// row's first key and ends at its last row's last one.
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
#include <algorithm>
#include <atomic>
#include <cstdint>
#include <mutex>

#include "../../include/attn.h"
#include "ctx_cache.h"
#include "internal.h"
#include "fp8.cuh"
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
// Both paths: 216 for each softmax warpgroup, 72 for the producer/MMA one
// (the split-KV instantiation spilled more with 224/56: 52 bytes against 8 at
// d = 128, and ran 1 % slower).
template <bool kKV>
constexpr int kRegsSoftmax = 216;
template <bool kKV>
constexpr int kRegsOther = 72;
static_assert(128 * (2 * kRegsSoftmax<true> + kRegsOther<true>) == kThreads * kRegsAtLaunch &&
                  128 * (2 * kRegsSoftmax<false> + kRegsOther<false>) == kThreads * kRegsAtLaunch,
              "register split must equal the launch allocation");
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: p <= 256 while m lags
// Largest overestimate (log2 units) of a tile's maximum logit allowed when a
// linear distance bias is bounded instead of applied before the maximum: the
// largest weight of the tile is then still >= 2^-96, far from fp32 underflow.
constexpr float kBiasBoundSlack = 96.0f;
// Bounded-wait limit handed to every launch (attn_set_wait_limit_ms).
std::atomic<uint64_t> g_wait_limit_ns{2000000000ull};

// Which of a row's 64 (even, odd) column pairs take the FMA-pipe exponential
// (exp2_poly_pair) instead of the MUFU one. bf16: one pair in four. Measured
// on the persistent kernel at (8, 32, 8192, 128, causal): 1/4 is 1 % faster
// than 3/8 below the power cap and 0.5 % under it, all-MUFU lies between,
// 1/2 is 5 % slower. FP8: the E4M3 MMAs take half the bf16 time, so the
// softmax is the longer leg by far and the FMA pipe has room for one pair in
// three (measured on the one-CTA-per-unit kernel: 1/3 beats 1/4 by 4 % and
// 1/2 is slower than both).
constexpr int kPolyPeriodF8 = 3;
template <bool kF8>
__host__ __device__ constexpr bool poly_pair(int cc) {
  if constexpr (kF8) return cc % kPolyPeriodF8 == kPolyPeriodF8 - 1;
  return (cc % 4) == 3;
}

// kF8: Q, K, V hold 8-bit E4M3 values (one byte each) instead of bf16.
template <int D, bool kF8 = false>
struct Cfg {
  static constexpr int kElemBytes = kF8 ? 1 : 2;
  static constexpr int kTileBytes = kTileRows * D * kElemBytes;  // one 128 x D tile
  static constexpr int kAtoms = D * kElemBytes / 128;   // 128-byte swizzle atoms per row
  static constexpr int kAtomBytes = kTileRows * 128;    // 16 KiB
  static constexpr int kStages = (kTileBytes == 32768) ? 4 : 8;  // tile slots of the ring
  // elements of the reduced dimension per MMA instruction (32 bytes of it)
  static constexpr int kMmaK = 32 / kElemBytes;
  static constexpr int kUnits = kStages / 2;           // (V, K) units in flight
  static constexpr int kQOff = 0;
  static constexpr int kRingOff = 2 * kTileBytes;
  static constexpr int kBarOff = kRingOff + kStages * kTileBytes;
  // q_full, kv_full[S], kv_empty[S], s_full[2], p_ready[2], o_final[2],
  // mma_done, q_empty (square path: the Q tiles may be overwritten),
  // stage_free (square path: the O staging tile may be overwritten)
  static constexpr int kNumBars = 1 + 2 * kStages + 6 + 3;
  static constexpr int kMiscOff = kBarOff + 8 * kNumBars;  // tmem base, abort flag
  // square path: one bf16 O tile (128 rows, 128-byte swizzle atoms of 64
  // columns) staged for its TMA store, after the barriers, 1024-aligned
  static constexpr int kStageOff = (kMiscOff + 16 + 1023) / 1024 * 1024;
  static constexpr int kStageBytes = kTileRows * D * 2;
  static constexpr int kSmemBytes = kStageOff + kStageBytes + 1024;  // + alignment slack
  static_assert(kSmemBytes <= 227 * 1024, "square path exceeds the shared memory of a CTA");
  // kv path: (m, l) of every softmax thread, swapped between the two
  // warpgroups when they took alternate KV tiles of one query tile
  static constexpr int kXchOff = kMiscOff + 16;
  static constexpr int kSmemBytesKv = kXchOff + 256 * 2 * 4 + 1024;
  static_assert(kSmemBytesKv <= 227 * 1024, "kv path exceeds the shared memory of a CTA");
  __host__ __device__ static constexpr uint32_t col_s(int g) { return g == 0 ? 0u : 128u; }
  __host__ __device__ static constexpr uint32_t col_o(int g) { return 256u + (g == 0 ? 0u : uint32_t(D)); }
};

struct FwdParams {
  void* o;
  float* lse;
  unsigned int* err;
  float v_descale;  // FP8 path: O is scaled by it (1 otherwise)
  int N, BH, nqb, T;  // N = keys (and query rows of the square problem); T = KV tiles
  // |scale| * log2(e) (times the FP8 descales); 0 when scale is 0, which
  // makes every allowed logit 0 (a uniform softmax over the allowed keys)
  float scale_log2;
  // tcgen05 instruction-descriptor bit that negates A (Q) in S = Q K^T: set
  // when scale < 0, so the softmax always multiplies by a positive factor
  uint32_t qk_negate;
  int causal;
  // square path: 1 when the work units are dealt in (heaviest, lightest)
  // pairs (more units than CTAs); 0: one unit per CTA
  int paired;
  uint64_t wait_limit_ns;
  // kv path only (Nq query rows against N keys, KV range split across CTAs)
  int Nq;
  int offset;    // N - Nq: causally, query row i is sequence position i + offset
  int nsplit;    // KV splits (1: O and lse written directly)
  int tps;       // KV tiles per split
  int alt;       // 1: one query tile per CTA, the two softmax warpgroups take alternate KV tiles
  float* part_o;    // [nsplit][BH][Nq][D] fp32, normalised per split (nsplit > 1)
  float* part_lse;  // [nsplit][BH][Nq] fp32 natural-log lse per split (nsplit > 1)
  int t_begin;      // first KV tile any query row needs (the splits cut [t_begin, T))
  int wl, wr;       // key window [pos - wl, pos + wr] around query position pos; < 0: unbounded
  int H;
  const float* slopes;  // per-head linear distance bias slopes (natural log units), or null
};

// What one CTA of the kv path works on.
struct KvWork {
  int split;
  int kv_lo;  // first KV tile of the split
  int na, nb; // KV tiles for softmax warpgroup a / b
};

// kv path: the (head, query block, KV split) of this CTA and the KV tiles each
// softmax warpgroup takes. Cheap integer arithmetic on blockIdx and the
// parameters, so the softmax warps recompute it for their epilogue instead of
// keeping it in registers through the main loop.
__device__ __forceinline__ KvWork kv_work_of(const FwdParams& p, int& bh, int& q0) {
  KvWork kw{0, 0, 0, 0};
  // (bh, split, query block), query blocks fastest; a block is one query
  // tile when alt, else two.
  const int per_bh = p.nqb * p.nsplit;
  bh = blockIdx.x / per_bh;
  const int rem = blockIdx.x % per_bh;
  kw.split = rem / p.nqb;
  const int r = rem % p.nqb;
  const int qblk = p.causal ? (p.nqb - 1 - r) : r;
  q0 = qblk * (p.alt ? kTileRows : kBlockRows);
  const int s_lo = p.t_begin + kw.split * p.tps;  // this split's KV tiles [s_lo, s_hi)
  const int s_hi = min(p.T, s_lo + p.tps);
  // one past the last KV tile that some row of the tile starting at r0 sees
  auto need = [&](int r0) -> int {
    if (r0 >= p.Nq) return 0;
    const int r1 = min(r0 + kTileRows - 1, p.Nq - 1);
    long long hi = p.N - 1;
    if (p.causal) hi = min(hi, static_cast<long long>(r1) + p.offset);
    if (p.wr >= 0) hi = min(hi, static_cast<long long>(r1) + p.offset + p.wr);
    return hi < 0 ? 0 : static_cast<int>(hi / kTileRows) + 1;
  };
  // first KV tile the first row of the CTA sees (a left window bound)
  const long long first_key =
      p.wl >= 0 ? max(0ll, static_cast<long long>(q0) + p.offset - p.wl) : 0ll;
  kw.kv_lo = max(s_lo, static_cast<int>(first_key / kTileRows));
  if (p.alt) {
    const int n = max(0, min(s_hi, need(q0)) - kw.kv_lo);
    kw.na = (n + 1) / 2;
    kw.nb = n / 2;
  } else {
    kw.na = max(0, min(s_hi, need(q0)) - kw.kv_lo);
    kw.nb = max(0, min(s_hi, need(q0 + kTileRows)) - kw.kv_lo);
  }
  return kw;
}

// Stores 32 consecutive output columns of one row: fp32 (a split's partial
// result) or bf16 (the final O).
template <int D>
__device__ __forceinline__ void store_row_chunk(const FwdParams& p, bool partial, size_t row_index,
                                                int col, const float (&v)[32]) {
  if (partial) {
    float4* dst = reinterpret_cast<float4*>(p.part_o + row_index * D + col);
#pragma unroll
    for (int u = 0; u < 8; ++u) dst[u] = make_float4(v[4 * u], v[4 * u + 1], v[4 * u + 2], v[4 * u + 3]);
  } else {
    uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.o) + row_index * D + col);
#pragma unroll
    for (int u = 0; u < 4; ++u)
      dst[u] = make_uint4(pack_bf16x2(v[8 * u], v[8 * u + 1]), pack_bf16x2(v[8 * u + 2], v[8 * u + 3]),
                          pack_bf16x2(v[8 * u + 4], v[8 * u + 5]), pack_bf16x2(v[8 * u + 6], v[8 * u + 7]));
  }
}

// ctl: shared address of the control barriers s_full[2], p_ready[2],
// o_final[2] (consecutive). kWin (square path): per-row key ranges as on the
// kv path, KV tiles counted from kv_lo.
// s_phase0: steps this warpgroup has taken before (the square path's work
// units follow one another on the same barriers); o_phase: parity of this
// unit's o_final phase. Returns false once a wait has given up.
template <int D, bool kKV, bool kF8 = false, bool kBias = kKV, bool kWin = false>
__device__ __forceinline__ bool softmax_role(const FwdParams& p, uint32_t tmem, uint32_t ctl,
                                             int bh, int q0, int n_kv, int g,
                                             const Watchdog& wd, int kv_lo, uint32_t s_phase0 = 0,
                                             uint32_t o_phase = 0,
                                             const CUtensorMap* tmap_o = nullptr,
                                             uint32_t stage = 0, uint32_t stage_use = 0) {
  using C = Cfg<D, kF8>;
  const int warp = threadIdx.x / 32;
  const int tid = threadIdx.x % 128;
  const uint32_t lane_base = static_cast<uint32_t>(32 * (warp % 4)) << 16;
  const uint32_t tS = tmem + lane_base + C::col_s(g);
  const uint32_t tO = tmem + lane_base + C::col_o(g);
  const uint32_t bar_s_full = ctl + 8u * g;
  const uint32_t bar_p_ready = ctl + 8u * (2 + g);
  const uint32_t bar_o_final = ctl + 8u * (4 + g);
  // kv path with alternate KV tiles: both warpgroups hold the same query rows
  const bool alt = kKV && p.alt;
  const int row_start = alt ? q0 : q0 + kTileRows * g;
  const int row = row_start + tid;
  // scale 0: allowed logits are replaced by 0 and masked ones stay -inf, then
  // scaled by 1 (scaling -inf by 0 would give NaN)
  const bool zero_scale = p.scale_log2 == 0.0f;
  const float c = zero_scale ? 1.0f : p.scale_log2;
  // kv path and windows: this row's allowed keys [key_lo, key_hi] (causal
  // limit, window, key count); the tile's first row has the lowest key_hi and
  // its last row the highest key_lo, which decide whether a KV tile needs
  // masking at all.
  constexpr bool kRange = kKV || kWin;
  int key_lo = 0, key_hi = p.N - 1, tile_hi = p.N - 1, tile_lo = 0;
  float slope_l2 = 0.0f;
  if constexpr (kRange) {
    auto hi_of = [&](int r) {
      long long h = p.N - 1;
      if (p.causal) h = min(h, static_cast<long long>(r) + p.offset);
      if (p.wr >= 0) h = min(h, static_cast<long long>(r) + p.offset + p.wr);
      return static_cast<int>(max(h, -1ll));
    };
    auto lo_of = [&](int r) {
      return p.wl >= 0 ? static_cast<int>(min(max(0ll, static_cast<long long>(r) + p.offset - p.wl),
                                              static_cast<long long>(p.N)))
                       : 0;
    };
    key_hi = hi_of(row);
    key_lo = lo_of(row);
    tile_hi = hi_of(row_start);
    tile_lo = lo_of(row_start + kTileRows - 1);
  }
  if (kBias && p.slopes) slope_l2 = p.slopes[bh % p.H] * 1.4426950408889634f;
  // sequence position of query row 0 (keys start at position 0)
  const int pos_offset = kKV ? p.offset : 0;

  float m_run = -INFINITY;
  float l_run = 0.0f;
  bool ok = true;
  for (int j = 0; j < n_kv; ++j) {
    if (!(ok = warp_wait(bar_s_full, (s_phase0 + j) & 1, wd))) break;
    tc_fence_after_sync();
    uint32_t sr[128];
    tmem_ld_x128_wait(tS, sr);

    bool need_mask;
    int col0;
    float cs = c;  // multiplier from the values in sr to log2-domain logits
    // distance bias on a tile wholly on one side of every row's position:
    // b(cc) = bias_b0 + bias_dk * cc (log2 units), applied in the exponent
    // rather than to sr
    bool bias_linear = false;
    float bias_b0 = 0.0f, bias_dk = 0.0f;
    if constexpr (kRange) {
      col0 = (kv_lo + (alt ? 2 * j + g : j)) * kTileRows;
      need_mask = (col0 + kTileRows - 1 > tile_hi) || (col0 < tile_lo) || zero_scale;
      if (need_mask) {
        const int lim_hi = key_hi - col0;
        const int lim_lo = key_lo - col0;
#pragma unroll
        for (int cc = 0; cc < 128; ++cc)
          sr[cc] = (cc > lim_hi || cc < lim_lo) ? 0xff800000u : (zero_scale ? 0u : sr[cc]);  // -inf
      }
    } else {
      col0 = j * kTileRows;
      need_mask =
          (p.causal && col0 + kTileRows - 1 > row_start) || (col0 + kTileRows > p.N) || zero_scale;
      if (need_mask) {
        int lim = p.N - 1 - col0;
        if (p.causal) lim = min(lim, row - col0);
#pragma unroll
        for (int cc = 0; cc < 128; ++cc)
          sr[cc] = cc > lim ? 0xff800000u : (zero_scale ? 0u : sr[cc]);  // -inf
      }
    }
    if (kBias && p.slopes) {
      // linear distance bias: x = s * c - slope * log2(e) * |pos - key|
      const float rel = static_cast<float>(row + pos_offset - col0);  // pos - col0
      // key <= pos for every unmasked key of the tile: a tile left of every
      // row's position, or any tile of a causal problem (the keys past a
      // row's position are -inf whatever is added to them)
      const bool left = p.causal || col0 + kTileRows - 1 <= row_start + pos_offset;
      const bool right = col0 >= row_start + kTileRows - 1 + pos_offset;  // key >= pos everywhere
      if ((left || right) && slope_l2 * (kTileRows - 1) <= kBiasBoundSlack) {
        // One side of every row's position: the bias is linear in the
        // column, b(cc) = b0 + dk * cc. The scores stay unbiased here; the
        // row maximum is bounded by max(s) * c + max(b) (max(b) over the
        // whole tile, masked columns included, so the bound may exceed the
        // row's largest logit by up to the bias range, at most the slack)
        // and the bias enters the exponent's FMA (below), one packed add per
        // pair.
        bias_dk = left ? slope_l2 : -slope_l2;
        bias_b0 = -bias_dk * rel;
        bias_linear = true;
      } else {
#pragma unroll
        for (int cc = 0; cc < 128; ++cc)
          sr[cc] = __float_as_uint(
              fmaf(__uint_as_float(sr[cc]), c, -slope_l2 * fabsf(rel - static_cast<float>(cc))));
        cs = 1.0f;  // sr now holds the biased log2-domain logits
      }
    }

    float mx[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) mx[u] = __uint_as_float(sr[u]);
#pragma unroll
    for (int cc = 8; cc < 128; cc += 2)
      mx[(cc / 2) % 8] = fmax3(mx[(cc / 2) % 8], __uint_as_float(sr[cc]), __uint_as_float(sr[cc + 1]));
    const float rmax = fmax3(fmax3(mx[0], mx[1], mx[2]), fmax3(mx[3], mx[4], mx[5]),
                             fmaxf(mx[6], mx[7]));
    // with a linear bias left out of sr, rmax * c + max(b) bounds the tile's
    // largest logit from above: p = 2^(x - m) <= 1 stays true when m is
    // raised to it, and the result is the exact softmax whatever m is
    const float m_tile =
        bias_linear ? fmaf(rmax, cs, fmaxf(bias_b0, fmaf(bias_dk, kTileRows - 1, bias_b0))) : rmax * cs;
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
    // pairs poly_pair picks on the FMA pipe (exp2_poly_pair). A linear bias
    // rides in the addend: (b(cc) - m, b(cc + 1) - m), stepped by 2 dk.
    const uint64_t c2 = f2_pack(cs, cs);
    uint64_t nm2 = bias_linear ? f2_pack(bias_b0 + neg_m, bias_b0 + bias_dk + neg_m)
                               : f2_pack(neg_m, neg_m);
    const uint64_t bias_step2 = f2_pack(2.0f * bias_dk, 2.0f * bias_dk);
    uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
    // P in tensor memory: bf16 pairs (64 columns) or, for FP8, four E4M3
    // values per column (32 columns; p <= 2^8 fits E4M3's range of 448)
    uint32_t pk[kF8 ? 32 : 64];
#pragma unroll
    for (int cc = 0; cc < 64; ++cc) {
      float x0, x1, p0, p1;
      f2_unpack(f2_fma(f2_pack(__uint_as_float(sr[2 * cc]), __uint_as_float(sr[2 * cc + 1])), c2, nm2),
                x0, x1);
      if (bias_linear) nm2 = f2_add(nm2, bias_step2);
      if (poly_pair<kF8>(cc)) {
        exp2_poly_pair(x0, x1, p0, p1);
      } else {
        p0 = ex2_approx(x0);
        p1 = ex2_approx(x1);
      }
      acc[cc % 4] = f2_add(acc[cc % 4], f2_pack(p0, p1));
      if constexpr (kF8) {
        const uint32_t h = pack_e4m3x2(p0, p1);
        if (cc % 2 == 0)
          pk[cc / 2] = h;
        else
          pk[cc / 2] |= h << 16;
      } else {
        pk[cc] = pack_bf16x2(p0, p1);
      }
    }
    if constexpr (kF8) {
      tmem_st_x32(tS, pk);
    } else {
      tmem_st_x64(tS, pk);
    }
    tmem_st_wait();
    tc_fence_before_sync();
    mbar_arrive(bar_p_ready);
    {
      float lo, hi;
      f2_unpack(f2_add(f2_add(acc[0], acc[1]), f2_add(acc[2], acc[3])), lo, hi);
      l_run += lo + hi;
    }
  }
  if constexpr (!kKV) {
    if (ok) ok = warp_wait(bar_o_final, o_phase, wd);
    if (!ok) return false;
    tc_fence_after_sync();

    // Epilogue: O / l -> bf16 (times V's scale on the FP8 path), lse in natural
    // log. The O tile goes through a shared staging tile (128-byte swizzle,
    // so the row-per-thread writes are free of bank conflicts) and leaves in
    // TMA stores of whole lines; writing rows straight from registers cost
    // ~16 partial-line stores per thread, thousands of cycles per tile. Both
    // query tiles and all work units of the CTA share the staging tile, in
    // turn: use u waits until the store of use u - 1 has read it.
    const float inv_l = kF8 ? p.v_descale / l_run : 1.0f / l_run;
    const bool valid = row < p.N;
    const uint32_t bar_stage_free = ctl + 64u;
    if (stage_use > 0 && !warp_wait(bar_stage_free, (stage_use - 1) & 1, wd)) return false;
    uint8_t* stage_ptr = nullptr;
    {
      extern __shared__ uint8_t smem_raw[];
      stage_ptr = smem_raw + (stage - smem_u32(smem_raw));
    }
#pragma unroll
    for (int ch = 0; ch < D / 32; ++ch) {
      uint32_t orr[32];
      tmem_ld_x32_wait(tO + ch * 32, orr);
      uint32_t w[16];
#pragma unroll
      for (int u = 0; u < 16; ++u)
        w[u] = pack_bf16x2(__uint_as_float(orr[2 * u]) * inv_l, __uint_as_float(orr[2 * u + 1]) * inv_l);
      // 16-byte chunk q of the row's 64-column atom goes to chunk q ^ (row & 7)
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int chunk = (ch % 2) * 4 + q;
        *reinterpret_cast<uint4*>(stage_ptr + (ch / 2) * (kTileRows * 128) + tid * 128 +
                                  ((chunk ^ (tid & 7)) * 16)) =
            make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
      }
    }
    fence_proxy_async_smem();
    named_barrier_sync(2 + g, 128);
    if (tid == 0) {
      // rows past N are clipped by the store
#pragma unroll
      for (int a = 0; a < D / 64; ++a)
        tma_store_3d(tmap_o, stage + a * (kTileRows * 128), a * 64, row_start, bh);
      bulk_commit();
      bulk_wait_read<0>();
      mbar_arrive(bar_stage_free);
    }
    if (valid) {
      const float m_fin = (m_run == -INFINITY) ? 0.0f : m_run;
      p.lse[static_cast<size_t>(bh) * p.N + row] = (m_fin + __log2f(l_run)) * 0.69314718055994531f;
    }
  } else {
    // A row that saw no unmasked key in this KV range (possible only when the
    // range is a split that starts past the row's causal limit): l = 0, which
    // gives O = 0 and lse = -inf, the neutral element of the combine.
    if (m_run == -INFINITY) l_run = 0.0f;
    int bh_unused, q0_unused;
    const KvWork kw = kv_work_of(p, bh_unused, q0_unused);
    const bool valid = row < p.Nq;
    const bool partial = p.nsplit > 1;
    const size_t row_index =
        (partial ? static_cast<size_t>(kw.split) * p.BH + bh : static_cast<size_t>(bh)) * p.Nq + row;
    float* lse_dst = partial ? p.part_lse : p.lse;
    const uint32_t bar_o_final0 = ctl + 8u * 4;
    if (!alt) {
      if (ok && n_kv > 0) ok = warp_wait(bar_o_final, 0, wd);
      if (!ok) return false;
      tc_fence_after_sync();
      const float inv_l = l_run > 0.0f ? 1.0f / l_run : 0.0f;
#pragma unroll
      for (int ch = 0; ch < D / 32; ++ch) {
        float v[32];
        if (n_kv > 0) {
          uint32_t orr[32];
          tmem_ld_x32_wait(tO + ch * 32, orr);
#pragma unroll
          for (int u = 0; u < 32; ++u) v[u] = __uint_as_float(orr[u]) * inv_l;
        } else {
#pragma unroll
          for (int u = 0; u < 32; ++u) v[u] = 0.0f;
        }
        if (valid) store_row_chunk<D>(p, partial, row_index, ch * 32, v);
      }
      if (valid)
        lse_dst[row_index] = l_run > 0.0f ? (m_run + __log2f(l_run)) * 0.69314718055994531f : -INFINITY;
    } else {
      // Both warpgroups hold the same rows: O = (O_a 2^(m_a-m) + O_b 2^(m_b-m)) /
      // (l_a 2^(m_a-m) + l_b 2^(m_b-m)) with m = max(m_a, m_b). Each warpgroup
      // waits for both accumulators, swaps (m, l) through shared memory and
      // writes half of the columns. Every softmax thread reaches the named
      // barrier, also after a failed wait, and all leave together if any wait
      // failed (a failed wait always sets the CTA's abort flag).
      if (ok && kw.na > 0) ok = warp_wait(bar_o_final0, 0, wd);
      if (ok && kw.nb > 0) ok = warp_wait(bar_o_final0 + 8u, 0, wd);
      extern __shared__ uint8_t smem_raw[];
      const uint32_t raw = smem_u32(smem_raw);
      float* xch = reinterpret_cast<float*>(smem_raw + (((raw + 1023u) & ~1023u) - raw) + C::kXchOff);
      xch[2 * (128 * g + tid)] = m_run;
      xch[2 * (128 * g + tid) + 1] = l_run;
      named_barrier_sync(1, 256);
      if (*wd.abort) return false;
      tc_fence_after_sync();
      const float m_o = xch[2 * (128 * (1 - g) + tid)];
      const float l_o = xch[2 * (128 * (1 - g) + tid) + 1];
      const float m_a = g == 0 ? m_run : m_o, l_a = g == 0 ? l_run : l_o;
      const float m_b = g == 0 ? m_o : m_run, l_b = g == 0 ? l_o : l_run;
      const float m = fmaxf(m_a, m_b);
      const float sa = l_a > 0.0f ? ex2_approx(m_a - m) : 0.0f;
      const float sb = l_b > 0.0f ? ex2_approx(m_b - m) : 0.0f;
      const float L = l_a * sa + l_b * sb;
      const float inv_L = L > 0.0f ? 1.0f / L : 0.0f;
      const float wa = sa * inv_L, wb = sb * inv_L;
      const uint32_t tOa = tmem + lane_base + C::col_o(0);
      const uint32_t tOb = tmem + lane_base + C::col_o(1);
#pragma unroll
      for (int ch = 0; ch < D / 64; ++ch) {
        const int col = g * (D / 2) + ch * 32;
        float v[32];
#pragma unroll
        for (int u = 0; u < 32; ++u) v[u] = 0.0f;
        if (kw.na > 0) {
          uint32_t orr[32];
          tmem_ld_x32_wait(tOa + col, orr);
#pragma unroll
          for (int u = 0; u < 32; ++u) v[u] = __uint_as_float(orr[u]) * wa;
        }
        if (kw.nb > 0) {
          uint32_t orr[32];
          tmem_ld_x32_wait(tOb + col, orr);
#pragma unroll
          for (int u = 0; u < 32; ++u) v[u] = fmaf(__uint_as_float(orr[u]), wb, v[u]);
        }
        if (valid) store_row_chunk<D>(p, partial, row_index, col, v);
      }
      if (valid && g == 0)
        lse_dst[row_index] = L > 0.0f ? (m + __log2f(L)) * 0.69314718055994531f : -INFINITY;
    }
  }
  return ok;
}

// Square path work units. The query blocks (256 rows) of a head are paired
// heaviest with lightest, (nqb - 1 - i, i): causally every pair then costs the
// same number of KV steps, so dealing the pairs to the CTAs in turn (CTA c
// takes pairs c, c + gridDim.x, ...) balances the SMs without a global work
// counter, and pairs are head-major so the CTAs running at the same time share
// K/V in L2. Unit k of the CTA is half k % 2 of its pair k / 2 (the heavy
// block first); with nqb odd the middle block of a head forms a pair alone.
// With no more units than SMs (p.paired = 0) each CTA takes the one unit
// blockIdx.x instead. Every role of the CTA walks the same sequence.
// With a key window (kWin) a unit starts at KV tile j0, the tile of the first
// key its first row may see, and na / nb count tiles from there; without one
// j0 = 0.
struct SquareUnit {
  int bh, q0, na, nb, j0;
};

// The KV tiles of the unit at q0: [j0, j0 + na) for query tile a and
// [j0, j0 + nb) for tile b (nb - na is 0 or 1).
template <bool kWin>
__device__ __forceinline__ void square_range(const FwdParams& p, SquareUnit& u) {
  if constexpr (kWin) {
    // one past the last KV tile that row r sees (causal limit, right window
    // bound, key count)
    auto end_of = [&](int r) {
      long long hi = p.N - 1;
      if (p.causal) hi = min(hi, static_cast<long long>(r));
      if (p.wr >= 0) hi = min(hi, static_cast<long long>(r) + p.wr);
      return static_cast<int>(hi / kTileRows) + 1;
    };
    u.j0 = (p.wl >= 0 ? max(0, u.q0 - p.wl) : 0) / kTileRows;
    u.na = end_of(u.q0 + kTileRows - 1) - u.j0;
    u.nb = end_of(u.q0 + kBlockRows - 1) - u.j0;
  } else {
    u.j0 = 0;
    u.na = p.causal ? min(p.T, u.q0 / kTileRows + 1) : p.T;
    u.nb = p.causal ? min(p.T, u.q0 / kTileRows + 2) : p.T;
  }
}

// k: the CTA's unit index, advanced past a skipped (absent) second half.
template <bool kWin = false>
__device__ __forceinline__ bool square_unit(const FwdParams& p, int& k, SquareUnit& u) {
  if (!p.paired) {
    // one wave: unit blockIdx.x alone
    if (k > 0 || static_cast<int>(blockIdx.x) >= p.nqb * p.BH) return false;
    u.bh = blockIdx.x / p.nqb;
    const int r = blockIdx.x % p.nqb;
    u.q0 = (p.causal ? p.nqb - 1 - r : r) * kBlockRows;
    square_range<kWin>(p, u);
    return true;
  }
  const int npairs = (p.nqb + 1) / 2;
  while (true) {
    const int pair = static_cast<int>(blockIdx.x) + (k / 2) * static_cast<int>(gridDim.x);
    if (pair >= npairs * p.BH) return false;
    const int i = pair % npairs;
    const int qblk = (k % 2 == 0) ? p.nqb - 1 - i : i;
    if (k % 2 == 1 && qblk == p.nqb - 1 - i) {  // the middle block of an odd nqb
      ++k;
      continue;
    }
    u.bh = pair / npairs;
    u.q0 = qblk * kBlockRows;
    square_range<kWin>(p, u);
    return true;
  }
}

// Square path producer. The ring runs on across the CTA's work units: ring
// unit 0 holds K_0 of the first unit; for each unit, ring units 1..nb hold
// (V_{u-1}, K_u), and its last one holds V_{nb-1} with K_0 of the next unit
// in the otherwise empty K half, so the next unit's first Q K^T needs no
// ring unit of its own. The next unit's Q tiles are loaded once the current
// unit's last Q K^T has completed (q_empty). Tile indices count from the
// unit's j0.
template <int D, bool kF8 = false, bool kWin = false>
__device__ __forceinline__ void producer_role(const CUtensorMap* tq, const CUtensorMap* tk,
                                              const CUtensorMap* tv, uint32_t base, uint32_t bars,
                                              const FwdParams& p, const Watchdog& wd) {
  using C = Cfg<D, kF8>;
  const uint32_t sQ = base + C::kQOff;
  const uint32_t sRing = base + C::kRingOff;
  const uint32_t bar_q = bars;
  const uint32_t bar_q_empty = bars + 8u * (1 + 2 * C::kStages + 7);
  const uint64_t pol_q = l2_policy_evict_first();
  const uint64_t pol_kv = l2_policy_evict_last();
  auto load_tile = [&](int slot, const CUtensorMap* map, int row, int bh, uint32_t bar_full) {
#pragma unroll
    for (int a = 0; a < C::kAtoms; ++a)
      tma_load_3d_hint(sRing + slot * C::kTileBytes + a * C::kAtomBytes, map, bar_full, a * 64, row, bh,
                       pol_kv);
  };
  auto load_q = [&](const SquareUnit& u) {
    mbar_arrive_expect_tx(bar_q, 2 * C::kTileBytes);
#pragma unroll
    for (int g = 0; g < 2; ++g)
#pragma unroll
      for (int a = 0; a < C::kAtoms; ++a)
        tma_load_3d_hint(sQ + g * C::kTileBytes + a * C::kAtomBytes, tq, bar_q, a * 64,
                         u.q0 + g * kTileRows, u.bh, pol_q);
  };
  // fills ring unit ug with the given tiles (row < 0: none) once its slot is free
  auto fill = [&](int ug, int v_row, int v_bh, int k_row, int k_bh) -> bool {
    const int us = ug % C::kUnits;
    const uint32_t bar_full = bars + 8u * (1 + us);
    if (!wait_one(bars + 8u * (1 + C::kStages + us), ((ug / C::kUnits) & 1) ^ 1u, wd)) return false;
    mbar_arrive_expect_tx(bar_full, (int(v_row >= 0) + int(k_row >= 0)) * C::kTileBytes);
    if (v_row >= 0) load_tile(2 * us, tv, v_row, v_bh, bar_full);
    if (k_row >= 0) load_tile(2 * us + 1, tk, k_row, k_bh, bar_full);
    return true;
  };
  int ug = 0;    // ring units filled so far
  int done = 0;  // work units of this CTA so far
  bool ok = true;
  int k = 0;
  SquareUnit cur;
  // first key row of a unit
  auto key0 = [](const SquareUnit& u) { return kWin ? u.j0 * kTileRows : 0; };
  if (square_unit<kWin>(p, k, cur)) {
    ok = fill(ug++, -1, 0, key0(cur), cur.bh);  // K_0 of the first unit
    if (ok) load_q(cur);
    while (ok) {
      int k2 = k + 1;
      SquareUnit nxt{0, 0, 0, 0, 0};
      const bool has_next = square_unit<kWin>(p, k2, nxt);
      const int nb = cur.nb;
      const int r0 = key0(cur);
      // the next unit's Q, K_0 and V_0 are fetched into L2 a few ring units
      // before this unit ends, so its first loads need not wait for HBM
      const int pf_at = max(1, nb - 3);
      for (int u = 1; ok && u <= nb; ++u) {
        if (u < nb)
          ok = fill(ug++, r0 + (u - 1) * kTileRows, cur.bh, r0 + u * kTileRows, cur.bh);
        else
          ok = fill(ug++, r0 + (u - 1) * kTileRows, cur.bh, has_next ? key0(nxt) : -1, nxt.bh);
        if (ok && u == pf_at && has_next) {
#pragma unroll
          for (int a = 0; a < C::kAtoms; ++a) {
            tma_prefetch_l2_3d(tq, a * 64, nxt.q0, nxt.bh);
            tma_prefetch_l2_3d(tq, a * 64, nxt.q0 + kTileRows, nxt.bh);
            tma_prefetch_l2_3d(tk, a * 64, key0(nxt), nxt.bh);
            tma_prefetch_l2_3d(tv, a * 64, key0(nxt), nxt.bh);
          }
        }
      }
      ++done;
      if (!ok || !has_next) break;
      // the next unit's Q once this unit's last Q K^T has completed
      if (!(ok = wait_one(bar_q_empty, (done - 1) & 1, wd))) break;
      load_q(nxt);
      k = k2;
      cur = nxt;
    }
  }
  // Teardown: every copy this thread issued must have landed before exit.
  if (done > 0) drain_wait(bar_q, (done - 1) & 1, wd);
  for (int w = (ug > C::kUnits ? ug - C::kUnits : 0); w < ug; ++w)
    drain_wait(bars + 8u * (1 + w % C::kUnits), (w / C::kUnits) & 1, wd);
}

template <int D, bool kF8 = false, bool kWin = false>
__device__ __forceinline__ void mma_role(uint32_t tmem, uint32_t base, uint32_t bars,
                                         const FwdParams& p, const Watchdog& wd) {
  const uint32_t qk_negate = p.qk_negate;
  using C = Cfg<D, kF8>;
  const uint32_t sQ = base + C::kQOff;
  const uint32_t sRing = base + C::kRingOff;
  const uint32_t bar_q = bars;
  const uint32_t bar_s_full0 = bars + 8u * (1 + 2 * C::kStages);
  const uint32_t bar_p_ready0 = bar_s_full0 + 16u;
  const uint32_t bar_o_final0 = bar_s_full0 + 32u;
  const uint32_t bar_mma_done = bar_s_full0 + 48u;
  const uint32_t idesc_qk =
      (kF8 ? idesc_e4m3_f32(128, 128, 0, 0) : idesc_bf16_f32(128, 128, 0, 0)) | qk_negate;
  constexpr uint32_t idesc_pv = kF8 ? idesc_e4m3_f32(128, D, 0, 1) : idesc_bf16_f32(128, D, 0, 1);

  // unit u (see producer_role): V_{u-1} in tile slot 2 (u % kUnits), K_u in the next one
  auto par_of = [](int u) { return static_cast<uint32_t>((u / C::kUnits) & 1); };
  auto full_bar = [&](int u) { return bars + 8u * (1 + u % C::kUnits); };
  auto empty_bar = [&](int u) { return bars + 8u * (1 + C::kStages + u % C::kUnits); };
  auto v_slot = [](int u) { return 2 * (u % C::kUnits); };
  auto k_slot = [](int u) { return 2 * (u % C::kUnits) + 1; };

  // S_g = Q_g K^T : A = Q tile (K-major), B = K tile (K-major); each
  // instruction reduces 32 bytes of d (16 bf16 or 32 E4M3 values), stepping
  // through the 128-byte swizzle atoms of a row.
  // The shared-memory descriptors of one launch differ only in their start
  // address (the low word; the high word holds the stride, version and
  // swizzle): keep the low words of the three bases, add each operand's
  // offset to them and attach the common high word, a few integer operations
  // per MMA for the single issuing thread.
  const uint64_t kk_hi = sdesc_sw128(0, 16, 1024) & 0xFFFFFFFF00000000ull;
  const uint32_t q_lo = static_cast<uint32_t>(sdesc_sw128(sQ, 16, 1024));
  const uint32_t r_lo = static_cast<uint32_t>(sdesc_sw128(sRing, 16, 1024));
  const uint32_t v_lo = static_cast<uint32_t>(sdesc_sw128(sRing, C::kAtomBytes, 1024));
  auto mk = [&](uint32_t lo) { return kk_hi | lo; };
  auto issue_qk = [&](int g, int slot) {
    // the opaque move keeps the compiler from hoisting every Q descriptor of
    // the unit loop into registers (the issuing warp has few to spare)
    uint32_t a0;
    asm volatile("mov.b32 %0, %1;" : "=r"(a0) : "r"(q_lo + static_cast<uint32_t>((g * C::kTileBytes) >> 4)));
    const uint32_t b0 = r_lo + static_cast<uint32_t>((slot * C::kTileBytes) >> 4);
#pragma unroll
    for (int kk = 0; kk < D / C::kMmaK; ++kk) {
      const uint32_t off = ((kk >> 2) * C::kAtomBytes + (kk & 3) * 32) >> 4;
      if constexpr (kF8)
        mma_ss_f8(tmem + C::col_s(g), mk(a0 + off), mk(b0 + off), idesc_qk, kk > 0 ? 1u : 0u);
      else
        mma_ss(tmem + C::col_s(g), mk(a0 + off), mk(b0 + off), idesc_qk, kk > 0 ? 1u : 0u);
    }
  };
  // O_g += P_g V : A = P in tensor memory (8 columns per instruction: 16 bf16
  // or 32 E4M3 keys), B = V tile (MN-major, rows of 128 bytes, one per key).
  auto issue_pv = [&](int g, int slot, bool accumulate) {
    const uint32_t b0 = v_lo + static_cast<uint32_t>((slot * C::kTileBytes) >> 4);
#pragma unroll
    for (int kk = 0; kk < kTileRows / C::kMmaK; ++kk) {
      if constexpr (kF8)
        mma_ts_f8(tmem + C::col_o(g), tmem + C::col_s(g) + kk * 8,
                  mk(b0 + static_cast<uint32_t>((kk * C::kMmaK * 128) >> 4)), idesc_pv,
                  (accumulate || kk > 0) ? 1u : 0u);
      else
        mma_ts(tmem + C::col_o(g), tmem + C::col_s(g) + kk * 8,
               mk(b0 + static_cast<uint32_t>((kk * 2048) >> 4)), idesc_pv,
               (accumulate || kk > 0) ? 1u : 0u);
    }
  };

  const uint32_t bar_q_empty = bar_s_full0 + 56u;
  int ug = 0;                // ring unit holding K_0 of the current work unit
  uint32_t pa = 0, pb = 0;   // P hand-offs of tile a / b taken so far
  int done = 0;              // work units of this CTA so far
  bool early_a = false;      // S_a(0) of the current unit already issued
  bool ok = true;
  int k = 0;
  SquareUnit cur;
  bool have = square_unit<kWin>(p, k, cur);
  while (ok && have) {
    const int na = cur.na, nb = cur.nb;
    int k2 = k + 1;
    SquareUnit nxt;
    const bool has_next = square_unit<kWin>(p, k2, nxt);
    if (!(ok = wait_one(bar_q, done & 1, wd) && wait_one(full_bar(ug), par_of(ug), wd))) break;
    tc_fence_after_sync();
    if (!early_a) {
      issue_qk(0, k_slot(ug));
      mma_commit(bar_s_full0);
    }
    issue_qk(1, k_slot(ug));
    mma_commit(bar_s_full0 + 8u);
    if (nb == 1) mma_commit(bar_q_empty);  // the unit's last Q K^T
    // ring unit ug: K_0 (and the previous unit's last V): read by now
    mma_commit(empty_bar(ug));
    early_a = false;
    for (int j = 0; j < nb; ++j) {
      const int ru = ug + j + 1;  // V_j, and K_{j+1} (the last: K_0 of the next unit)
      if (!(ok = wait_one(full_bar(ru), par_of(ru), wd))) break;
      if (j < na) {
        if (!(ok = wait_spin(bar_p_ready0, pa & 1, wd))) break;
        ++pa;
        tc_fence_after_sync();
        issue_pv(0, v_slot(ru), j > 0);
        if (j + 1 < na) {
          issue_qk(0, k_slot(ru));
          mma_commit(bar_s_full0);
        } else {
          mma_commit(bar_o_final0);
        }
      }
      if (j + 1 == nb && has_next) {
        // tile b's last P is still being computed: tile a's first Q K^T of the
        // next unit goes as soon as the next Q tiles land, so that tile a's
        // softmax starts that unit while tile b finishes this one
        uint64_t t0 = 0;
        for (uint32_t it = 1;; ++it) {
          if (mbar_test_wait(bar_p_ready0 + 8u, pb & 1)) break;
          if (mbar_test_wait(bar_q, (done + 1) & 1)) {
            tc_fence_after_sync();
            issue_qk(0, k_slot(ru));
            mma_commit(bar_s_full0);
            early_a = true;
            break;
          }
          if ((it & 63) == 0) {
            if (t0 == 0) t0 = global_timer_ns();
            if (*wd.abort || timed_out(t0, wd)) {
              ok = false;
              break;
            }
          }
        }
        if (!ok) break;
      }
      if (!(ok = wait_spin(bar_p_ready0 + 8u, pb & 1, wd))) break;
      ++pb;
      tc_fence_after_sync();
      issue_pv(1, v_slot(ru), j > 0);
      if (j + 1 < nb) {
        issue_qk(1, k_slot(ru));
        mma_commit(bar_s_full0 + 8u);
        if (j + 2 == nb) mma_commit(bar_q_empty);  // the unit's last Q K^T
      } else {
        mma_commit(bar_o_final0 + 8u);
      }
      // the last ring unit also holds the next unit's K_0: released after
      // that unit's first Q K^T
      if (j + 1 < nb || !has_next) mma_commit(empty_bar(ru));
    }
    ug += nb;
    ++done;
    k = k2;
    cur = nxt;
    have = has_next;
  }
  // Teardown: all MMAs this thread issued must be complete before the tensor
  // memory is freed.
  mma_commit(bar_mma_done);
  drain_wait(bar_mma_done, 0, wd);
}

// kv path producer. Query rows q0.. (one tile when alt, else two), then K/V
// tiles of the CTA's range [kv_lo, kv_lo + n) in two-slot units:
//   shared (both query tiles see every KV tile): unit 0 = K_0, unit u >= 1 =
//     (V_{u-1}, K_u), unit n = V_{n-1} only;
//   alt (warpgroup a takes KV tiles 0, 2, 4, ..., b takes 1, 3, 5, ...):
//     unit 0 = (K_0, K_1), unit u >= 1 = (V_{u-1}, K_{u+1}).
// Tile indices are relative to kv_lo.
template <int D>
__device__ __forceinline__ void producer_role_kv(const CUtensorMap* tq, const CUtensorMap* tk,
                                                 const CUtensorMap* tv, uint32_t base,
                                                 uint32_t bars, int bh, int q0, int kv_lo, int n,
                                                 bool alt, bool kv_reuse, const Watchdog& wd) {
  using C = Cfg<D>;
  if (n == 0) return;
  const uint32_t sQ = base + C::kQOff;
  const uint32_t sRing = base + C::kRingOff;
  const uint32_t bar_q = bars;
  const uint64_t pol_q = l2_policy_evict_first();
  // with one query block per head every KV tile is read by exactly one CTA
  const uint64_t pol_kv = kv_reuse ? l2_policy_evict_last() : l2_policy_evict_first();
  const int nq = alt ? 1 : 2;

  mbar_arrive_expect_tx(bar_q, nq * C::kTileBytes);
  for (int g = 0; g < nq; ++g)
#pragma unroll
    for (int a = 0; a < C::kAtoms; ++a)
      tma_load_3d_hint(sQ + g * C::kTileBytes + a * C::kAtomBytes, tq, bar_q, a * 64,
                       q0 + g * kTileRows, bh, pol_q);

  int u = 0;
  for (; u <= n; ++u) {
    const int us = u % C::kUnits;
    const uint32_t ph = (u / C::kUnits) & 1;
    const uint32_t bar_full = bars + 8u * (1 + us);
    const uint32_t bar_empty = bars + 8u * (1 + C::kStages + us);
    if (!wait_one(bar_empty, ph ^ 1u, wd)) break;
    const CUtensorMap* map0 = nullptr;  // first slot of the unit
    const CUtensorMap* map1 = nullptr;  // second slot
    int t0 = 0, t1 = 0;
    if (alt) {
      if (u == 0) {
        map0 = tk;
        t0 = 0;
        if (n > 1) map1 = tk, t1 = 1;
      } else {
        map0 = tv;
        t0 = u - 1;
        if (u + 1 < n) map1 = tk, t1 = u + 1;
      }
    } else {
      if (u >= 1) map0 = tv, t0 = u - 1;
      if (u < n) map1 = tk, t1 = u;
    }
    mbar_arrive_expect_tx(bar_full, (int(map0 != nullptr) + int(map1 != nullptr)) * C::kTileBytes);
    if (map0) {
#pragma unroll
      for (int a = 0; a < C::kAtoms; ++a)
        tma_load_3d_hint(sRing + (2 * us) * C::kTileBytes + a * C::kAtomBytes, map0, bar_full,
                         a * 64, (kv_lo + t0) * kTileRows, bh, pol_kv);
    }
    if (map1) {
#pragma unroll
      for (int a = 0; a < C::kAtoms; ++a)
        tma_load_3d_hint(sRing + (2 * us + 1) * C::kTileBytes + a * C::kAtomBytes, map1, bar_full,
                         a * 64, (kv_lo + t1) * kTileRows, bh, pol_kv);
    }
  }
  drain_wait(bar_q, 0, wd);
  for (int w = (u > C::kUnits ? u - C::kUnits : 0); w < u; ++w)
    drain_wait(bars + 8u * (1 + w % C::kUnits), (w / C::kUnits) & 1, wd);
}

// kv path MMA issuer; the unit layout is the one producer_role_kv loads.
template <int D>
__device__ __forceinline__ void mma_role_kv(uint32_t tmem, uint32_t base, uint32_t bars, int na,
                                            int nb, bool alt, uint32_t qk_negate,
                                            const Watchdog& wd) {
  using C = Cfg<D>;
  const uint32_t sQ = base + C::kQOff;
  const uint32_t sRing = base + C::kRingOff;
  const uint32_t bar_q = bars;
  const uint32_t bar_s_full0 = bars + 8u * (1 + 2 * C::kStages);
  const uint32_t bar_p_ready0 = bar_s_full0 + 16u;
  const uint32_t bar_o_final0 = bar_s_full0 + 32u;
  const uint32_t bar_mma_done = bar_s_full0 + 48u;
  const uint32_t idesc_qk = idesc_bf16_f32(128, 128, 0, 0) | qk_negate;
  constexpr uint32_t idesc_pv = idesc_bf16_f32(128, D, 0, 1);

  auto par_of = [](int u) { return static_cast<uint32_t>((u / C::kUnits) & 1); };
  auto full_bar = [&](int u) { return bars + 8u * (1 + u % C::kUnits); };
  auto empty_bar = [&](int u) { return bars + 8u * (1 + C::kStages + u % C::kUnits); };
  auto slot0 = [](int u) { return 2 * (u % C::kUnits); };
  auto slot1 = [](int u) { return 2 * (u % C::kUnits) + 1; };

  // S_g = Q_qt K^T into tile g's S columns
  auto issue_qk = [&](int g, int qt, int slot) {
    const uint32_t a0 = sQ + qt * C::kTileBytes;
    const uint32_t b0 = sRing + slot * C::kTileBytes;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const uint32_t off = (kk >> 2) * C::kAtomBytes + (kk & 3) * 32;
      mma_ss(tmem + C::col_s(g), sdesc_sw128(a0 + off, 16, 1024), sdesc_sw128(b0 + off, 16, 1024),
             idesc_qk, kk > 0 ? 1u : 0u);
    }
  };
  auto issue_pv = [&](int g, int slot, bool accumulate) {
    const uint32_t b0 = sRing + slot * C::kTileBytes;
#pragma unroll
    for (int kk = 0; kk < kTileRows / 16; ++kk)
      mma_ts(tmem + C::col_o(g), tmem + C::col_s(g) + kk * 8,
             sdesc_sw128(b0 + kk * 2048, C::kAtomBytes, 1024), idesc_pv,
             (accumulate || kk > 0) ? 1u : 0u);
  };

  const int n = alt ? na + nb : max(na, nb);
  if (n > 0) {
    bool ok = wait_one(bar_q, 0, wd) && wait_one(full_bar(0), par_of(0), wd);
    if (ok) {
      tc_fence_after_sync();
      if (alt) {
        issue_qk(0, 0, slot0(0));
        mma_commit(bar_s_full0);
        if (nb > 0) {
          issue_qk(1, 0, slot1(0));
          mma_commit(bar_s_full0 + 8u);
        }
      } else {
        if (na > 0) {
          issue_qk(0, 0, slot1(0));
          mma_commit(bar_s_full0);
        }
        if (nb > 0) {
          issue_qk(1, 1, slot1(0));
          mma_commit(bar_s_full0 + 8u);
        }
      }
      mma_commit(empty_bar(0));
    }
    if (alt) {
      // unit u: V_{u-1} for warpgroup g = (u-1) % 2 (its step i = (u-1) / 2),
      // and K_{u+1}, that warpgroup's next KV tile
      for (int u = 1; ok && u <= n; ++u) {
        const int g = (u - 1) & 1;
        const int i = (u - 1) >> 1;
        if (!(ok = wait_one(full_bar(u), par_of(u), wd))) break;
        if (!(ok = wait_one(bar_p_ready0 + 8u * g, i & 1, wd))) break;
        tc_fence_after_sync();
        issue_pv(g, slot0(u), i > 0);
        if (u + 1 < n) {
          issue_qk(g, 0, slot1(u));
          mma_commit(bar_s_full0 + 8u * g);
        } else {
          mma_commit(bar_o_final0 + 8u * g);
        }
        mma_commit(empty_bar(u));
      }
    } else {
      for (int j = 0; ok && j < n; ++j) {
        const int u = j + 1;  // V_j and K_{j+1}
        if (!(ok = wait_one(full_bar(u), par_of(u), wd))) break;
#pragma unroll
        for (int g = 0; g < 2; ++g) {
          const int ng = g == 0 ? na : nb;
          if (j < ng) {
            if (!(ok = wait_one(bar_p_ready0 + 8u * g, j & 1, wd))) break;
            tc_fence_after_sync();
            issue_pv(g, slot0(u), j > 0);
            if (j + 1 < ng) {
              issue_qk(g, g, slot1(u));
              mma_commit(bar_s_full0 + 8u * g);
            } else {
              mma_commit(bar_o_final0 + 8u * g);
            }
          }
        }
        if (!ok) break;
        mma_commit(empty_bar(u));
      }
    }
  }
  mma_commit(bar_mma_done);
  drain_wait(bar_mma_done, 0, wd);
}

// kD: head dimension. kKV: the kv path (Nq query rows against N keys, the
// KV range of each head split across CTAs); false: the square problem.
// kF8 (square problem only): E4M3 Q, K, V and P. kBias: the distance bias
// (applied when p.slopes is set). kWin (square bf16 only): key windows.
template <int D, bool kKV, bool kF8 = false, bool kBias = kKV, bool kWin = false>
__global__ void __launch_bounds__(kThreads, 1)
    fused_attn_fwd_kernel(const __grid_constant__ CUtensorMap tmap_q,
                          const __grid_constant__ CUtensorMap tmap_k,
                          const __grid_constant__ CUtensorMap tmap_v,
                          const __grid_constant__ CUtensorMap tmap_o, const FwdParams p) {
  static_assert(!(kKV && kF8), "the FP8 path covers the square problem");
  static_assert(!(kWin && (kKV || kF8)), "kWin selects the windowed square bf16 path");
  using C = Cfg<D, kF8>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;  // 128B swizzle wants 1024-byte alignment
  uint8_t* smem = smem_raw + (base - raw);
  const uint32_t bars = base + C::kBarOff;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kMiscOff);
  volatile uint32_t* abort_flag = tmem_slot + 1;

  const int warp = threadIdx.x / 32;
  const uint32_t lane = threadIdx.x % 32;

  // Work: the kv path's CTA is one (head, key range, query block); a square
  // path CTA walks the work units blockIdx.x, blockIdx.x + gridDim.x, ...
  // (square_unit), one after another on the same barriers and buffers.
  int bh = 0, q0 = 0, na = 0, nb = 0;
  KvWork kw{0, 0, 0, 0};
  if constexpr (kKV) {
    kw = kv_work_of(p, bh, q0);
    na = kw.na;
    nb = kw.nb;
  }

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
    mbar_init(b6 + 56, 1);   // q_empty
    mbar_init(b6 + 64, 1);   // stage_free
    *abort_flag = 0u;
    mbar_fence_init();
  }
  if (warp == kProducerWarp && lane == 0) {
    tma_prefetch_desc(&tmap_q);
    tma_prefetch_desc(&tmap_k);
    tma_prefetch_desc(&tmap_v);
    if constexpr (!kKV) tma_prefetch_desc(&tmap_o);
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
    regs_increase<kRegsSoftmax<kKV>>();
    const int g = warp / 4;
    const uint32_t ctl = bars + 8u * (1 + 2 * C::kStages);
    if constexpr (kKV) {
      softmax_role<D, kKV, kF8, kBias>(p, tmem, ctl, bh, q0, g == 0 ? na : nb, g, wd, kw.kv_lo);
    } else {
      uint32_t steps = 0;  // this warpgroup's S hand-offs so far (s_full phases)
      uint32_t done = 0;   // work units so far (o_final phases)
      SquareUnit u;
      for (int k = 0; square_unit<kWin>(p, k, u); ++k, ++done) {
        const int n = g == 0 ? u.na : u.nb;
        if (!softmax_role<D, kKV, kF8, kBias, kWin>(p, tmem, ctl, u.bh, u.q0, n, g, wd,
                                                    kWin ? u.j0 : 0, steps, done & 1, &tmap_o,
                                                    base + C::kStageOff, 2 * done + g))
          break;
        steps += n;
      }
      // the O stores this warpgroup's leader issued complete before exit
      if (threadIdx.x % 128 == 0) bulk_wait_all();
    }
  } else {
    regs_decrease<kRegsOther<kKV>>();
    if constexpr (!kKV) {
      if (warp == kProducerWarp) {
        if (lane == 0) producer_role<D, kF8, kWin>(&tmap_q, &tmap_k, &tmap_v, base, bars, p, wd);
      } else if (warp == kMmaWarp) {
        if (lane == 0) mma_role<D, kF8, kWin>(tmem, base, bars, p, wd);
      }
    } else {
      const bool alt = p.alt != 0;
      if (warp == kProducerWarp) {
        if (lane == 0)
          producer_role_kv<D>(&tmap_q, &tmap_k, &tmap_v, base, bars, bh, q0, kw.kv_lo,
                              alt ? na + nb : max(na, nb), alt, p.nqb > 1, wd);
      } else if (warp == kMmaWarp) {
        if (lane == 0) mma_role_kv<D>(tmem, base, bars, na, nb, alt, p.qk_negate, wd);
      }
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

}  // namespace

bool current_context_id(unsigned long long* id) {
  using GetCurrent = CUresult (*)(CUcontext*);
  using GetId = CUresult (*)(CUcontext, unsigned long long*);
  static GetCurrent get_current = nullptr;
  static GetId get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<GetCurrent>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<GetId>(p);
  });
  if (!get_current || !get_id) return false;
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS) return false;
  if (ctx == nullptr) {
    // the runtime binds the device's primary context to this thread lazily
    if (cudaFree(nullptr) != cudaSuccess || get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr)
      return false;
  }
  return get_id(ctx, id) == CUDA_SUCCESS;
}

namespace {

unsigned int* device_error_word();

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

// [B*H, N, d] viewed as a 3-D tensor (d innermost) of bf16 (elem_bytes 2)
// or E4M3 bytes (elem_bytes 1); box = 128 bytes of a row (one swizzle atom:
// 64 bf16 or 128 E4M3) x 128 rows x 1 head; rows past N read as 0.
bool encode_qkv_map(CUtensorMap* m, const void* ptr, int BH, int N, int d, int elem_bytes = 2,
                    int box_rows = kTileRows) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N),
                        static_cast<cuuint64_t>(BH)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * elem_bytes,
                           static_cast<cuuint64_t>(N) * static_cast<cuuint64_t>(d) * elem_bytes};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(128 / elem_bytes),
                       static_cast<cuuint32_t>(box_rows), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(m, elem_bytes == 1 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                   3, const_cast<void*>(ptr), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace

bool encode_bf16_tiled_3d(CUtensorMap* m, const void* ptr, uint64_t d0, uint64_t d1, uint64_t d2,
                          uint32_t box0, uint32_t box1) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {d0 * 2, d0 * d1 * 2};
  cuuint32_t box[3] = {box0, box1, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

unsigned int* library_error_word() { return device_error_word(); }

namespace {

// Device address of g_device_error in the current context.
unsigned int* device_error_word() {
  static CtxCache<unsigned int*> cache;
  unsigned int* ptr = nullptr;
  if (!cache.get(&ptr, [](unsigned int** out) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_device_error) != cudaSuccess) return false;
        *out = static_cast<unsigned int*>(p);
        return true;
      }))
    return nullptr;
  return ptr;
}

// Multiprocessors of the current device, cached per context.
int sm_count_current() {
  static CtxCache<int> cache;
  int n = 0;
  if (!cache.get(&n, [](int* out) {
        int dev = 0;
        return cudaGetDevice(&dev) == cudaSuccess &&
               cudaDeviceGetAttribute(out, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess;
      }))
    return 0;
  return n;
}

// Once per (kernel, context): raise the kernel's dynamic shared-memory limit
// and check the register allocation the in-kernel register split relies on
// (the softmax warpgroups' setmaxnreg increase draws on exactly the launch
// allocation, so any other count could make it wait forever; the build also
// rejects such a binary). Later calls in the same context reuse that result.
template <auto Kernel>
int prepare_kernel(int smem_bytes) {
  static CtxCache<int> cache;
  int status = ATTN_ERR_CUDA;
  if (!cache.get(&status, [smem_bytes](int* out) {
        cudaFuncAttributes fa{};
        if (cudaFuncSetAttribute(Kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 smem_bytes) != cudaSuccess ||
            cudaFuncGetAttributes(&fa, Kernel) != cudaSuccess)
          return false;  // not cached: a later call may succeed
        *out = (fa.numRegs == kRegsAtLaunch && fa.maxThreadsPerBlock >= kThreads) ? ATTN_OK
                                                                                  : ATTN_ERR_LAUNCH;
        return true;
      }))
    return ATTN_ERR_CUDA;
  return status;
}

// One launch of a square-path instantiation, after its one-time preparation.
template <auto Kernel>
int launch_square(unsigned grid, int smem_bytes, cudaStream_t stream, const CUtensorMap& mq,
                  const CUtensorMap& mk, const CUtensorMap& mv, const CUtensorMap& mo,
                  const FwdParams& p) {
  const int prep = prepare_kernel<Kernel>(smem_bytes);
  if (prep != ATTN_OK) return prep;
  Kernel<<<grid, kThreads, smem_bytes, stream>>>(mq, mk, mv, mo, p);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_LAUNCH;
}

// kF8: Q, K, V are E4M3 with the given dequantisation scales (the scores get
// q_descale * k_descale, O gets v_descale); otherwise bf16 and all scales 1.
template <int D, bool kF8 = false>
int launch_fused_d(const AttnArgs& a, cudaStream_t stream, float q_descale = 1.0f,
                   float k_descale = 1.0f, float v_descale = 1.0f) {
  using C = Cfg<D, kF8>;
  const int BH = a.B * a.H;
  CUtensorMap mq, mk, mv;
  CUtensorMap mo;
  if (!encode_qkv_map(&mq, a.q, BH, a.N, D, C::kElemBytes) ||
      !encode_qkv_map(&mk, a.k, BH, a.N, D, C::kElemBytes) ||
      !encode_qkv_map(&mv, a.v, BH, a.N, D, C::kElemBytes) ||
      !encode_qkv_map(&mo, a.o, BH, a.N, D, 2))
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
  p.scale_log2 = static_cast<float>(std::fabs(static_cast<double>(a.scale)) * q_descale *
                                    k_descale * 1.4426950408889634);
  p.qk_negate = a.scale < 0.0f ? kIdescNegateA : 0u;
  p.v_descale = v_descale;
  p.causal = a.causal;
  p.wait_limit_ns = g_wait_limit_ns.load(std::memory_order_relaxed);
  p.H = a.H;
  p.slopes = a.slopes;
  p.wl = a.window_left;
  p.wr = a.window_right;
  const long long units = static_cast<long long>(p.nqb) * BH;
  if (units > 0x7fffffffLL) return ATTN_ERR_SHAPE;
  // persistent grid: one CTA per SM (one fits), each walking work units in
  // balanced pairs; with no more units than SMs, one unit per CTA (pairing
  // would only put two units behind each other on half the CTAs)
  const int sms = sm_count_current();
  if (sms < 1) return ATTN_ERR_CUDA;
  p.paired = units > sms ? 1 : 0;
  const unsigned grid = static_cast<unsigned>(std::min<long long>(units, sms));
  // the distance bias and the key windows have instantiations of their own,
  // so that the plain kernel's loops carry none of their arithmetic
  if constexpr (kF8) {
    return launch_square<fused_attn_fwd_kernel<D, false, true, false>>(grid, C::kSmemBytes, stream,
                                                                        mq, mk, mv, mo, p);
  } else {
    const bool bias = a.slopes != nullptr;
    if (a.window_left >= 0 || a.window_right >= 0)
      return bias ? launch_square<fused_attn_fwd_kernel<D, false, false, true, true>>(
                        grid, C::kSmemBytes, stream, mq, mk, mv, mo, p)
                  : launch_square<fused_attn_fwd_kernel<D, false, false, false, true>>(
                        grid, C::kSmemBytes, stream, mq, mk, mv, mo, p);
    return bias ? launch_square<fused_attn_fwd_kernel<D, false, false, true>>(grid, C::kSmemBytes,
                                                                             stream, mq, mk, mv, mo, p)
                : launch_square<fused_attn_fwd_kernel<D, false, false, false>>(
                      grid, C::kSmemBytes, stream, mq, mk, mv, mo, p);
  }
}

// ------------------------------------------------------------ kv path host

template <int D>
int launch_fused_kv_d(const AttnKvArgs& a, const KvPlan& plan, void* workspace,
                      cudaStream_t stream) {
  using C = Cfg<D>;
  const int BH = a.B * a.H;
  CUtensorMap mq, mk, mv;
  if (!encode_qkv_map(&mq, a.q, BH, a.Nq, D) || !encode_qkv_map(&mk, a.k, BH, a.Nk, D) ||
      !encode_qkv_map(&mv, a.v, BH, a.Nk, D))
    return ATTN_ERR_CUDA;
  unsigned int* err = device_error_word();
  if (!err) return ATTN_ERR_CUDA;
  FwdParams p{};
  p.o = a.o;
  p.lse = a.lse;
  p.err = err;
  p.N = a.Nk;
  p.BH = BH;
  p.nqb = plan.nqb;
  p.T = plan.T;
  p.scale_log2 = static_cast<float>(std::fabs(static_cast<double>(a.scale)) * 1.4426950408889634);
  p.qk_negate = a.scale < 0.0f ? kIdescNegateA : 0u;
  p.causal = a.causal;
  p.wait_limit_ns = g_wait_limit_ns.load(std::memory_order_relaxed);
  p.Nq = a.Nq;
  p.offset = a.Nk - a.Nq;
  p.nsplit = plan.nsplit;
  p.tps = plan.tps;
  p.alt = plan.alt;
  p.t_begin = plan.t_begin;
  p.wl = a.window_left;
  p.wr = a.window_right;
  p.H = a.H;
  p.slopes = a.slopes;
  if (plan.nsplit > 1) {
    p.part_o = static_cast<float*>(workspace);
    p.part_lse = reinterpret_cast<float*>(static_cast<char*>(workspace) +
                                          kv_partial_o_bytes(BH, a.Nq, D, plan.nsplit));
  }
  const long long grid = static_cast<long long>(plan.nqb) * plan.nsplit * BH;
  if (grid > 0x7fffffffLL) return ATTN_ERR_SHAPE;
  const int prep = prepare_kernel<fused_attn_fwd_kernel<D, true>>(C::kSmemBytesKv);
  if (prep != ATTN_OK) return prep;
  fused_attn_fwd_kernel<D, true>
      <<<static_cast<unsigned>(grid), kThreads, C::kSmemBytesKv, stream>>>(mq, mk, mv, mv, p);
  if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_LAUNCH;
  if (plan.nsplit > 1)
    return launch_lse_combine(p.part_o, p.part_lse, a.o, a.lse, BH * a.Nq, D, plan.nsplit, stream);
  return ATTN_OK;
}

}  // namespace

KvPlan plan_kv(int BH, int Nq, int Nk, int num_splits, int window_left) {
  KvPlan pl{};
  pl.T = (Nk + kTileRows - 1) / kTileRows;
  pl.alt = Nq <= kTileRows ? 1 : 0;
  pl.nqb = (Nq + (pl.alt ? kTileRows : kBlockRows) - 1) / (pl.alt ? kTileRows : kBlockRows);
  // keys before the first query row's window are never read: the splits cut
  // [t_begin, T) (query row 0 is sequence position Nk - Nq)
  const long long first_key =
      window_left >= 0 ? std::max(0ll, static_cast<long long>(Nk) - Nq - window_left) : 0ll;
  pl.t_begin = static_cast<int>(std::min<long long>(first_key / kTileRows, pl.T - 1));
  const int len = pl.T - pl.t_begin;
  const int s = std::max(1, std::min(num_splits, len));
  pl.tps = (len + s - 1) / s;
  pl.nsplit = (len + pl.tps - 1) / pl.tps;  // no empty split
  (void)BH;
  return pl;
}

int default_kv_splits(int BH, int Nq, int Nk, int sms, int window_left) {
  const KvPlan one = plan_kv(BH, Nq, Nk, 1, window_left);
  const long long base = static_cast<long long>(BH) * one.nqb;
  if (sms < 1 || base >= sms) return 1;
  // At least kMinTilesPerSplit KV tiles per CTA keeps the per-CTA start-up
  // (Q load, pipeline fill, epilogue) small against its streaming time.
  constexpr int kMinTilesPerSplit = 8;
  const int max_s = std::max(1, std::min(kMaxKvSplits, (one.T - one.t_begin) / kMinTilesPerSplit));
  auto eff = [&](int s) {
    const long long n = base * plan_kv(BH, Nq, Nk, s, window_left).nsplit;
    const long long waves = (n + sms - 1) / sms;
    return static_cast<double>(n) / static_cast<double>(waves * sms);
  };
  double best = 0.0;
  for (int s = 1; s <= max_s; ++s) best = std::max(best, eff(s));
  // the fewest splits within 15% of the best wave efficiency
  for (int s = 1; s <= max_s; ++s)
    if (eff(s) >= 0.85 * best) return plan_kv(BH, Nq, Nk, s, window_left).nsplit;
  return 1;
}

size_t kv_partial_o_bytes(int BH, int Nq, int d, int nsplit) {
  const size_t b = static_cast<size_t>(nsplit) * BH * Nq * d * sizeof(float);
  return (b + 255) & ~static_cast<size_t>(255);
}

size_t kv_workspace_bytes(int BH, int Nq, int d, int nsplit) {
  if (nsplit <= 1) return 0;
  return kv_partial_o_bytes(BH, Nq, d, nsplit) + static_cast<size_t>(nsplit) * BH * Nq * sizeof(float);
}

int launch_fused_kv(const AttnKvArgs& a, const KvPlan& plan, void* workspace, cudaStream_t stream) {
  return a.d == 128 ? launch_fused_kv_d<128>(a, plan, workspace, stream)
                    : launch_fused_kv_d<64>(a, plan, workspace, stream);
}

int launch_fused(const AttnArgs& a, cudaStream_t stream) {
  return a.d == 128 ? launch_fused_d<128>(a, stream) : launch_fused_d<64>(a, stream);
}

int launch_fused_fp8(const AttnArgs& a, float q_descale, float k_descale, float v_descale,
                     cudaStream_t stream) {
  return launch_fused_d<128, true>(a, stream, q_descale, k_descale, v_descale);
}

void set_wait_limit_ms(int ms) {
  g_wait_limit_ns.store(static_cast<uint64_t>(ms) * 1000000ull, std::memory_order_relaxed);
}

int wait_limit_ms() {
  return static_cast<int>(g_wait_limit_ns.load(std::memory_order_relaxed) / 1000000ull);
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
