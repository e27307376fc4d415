/*
 * attn.h - C ABI of the B200 (sm_100a) exact-attention forward library
 * (libattn_b200.so).
 *
 * The operation is exact scaled dot-product attention,
 *
 *     O = softmax(Q K^T * scale  [+ causal mask]) V,
 *
 * with the row-wise softmax and the three steps (scores, softmax, output) as
 * described on the grasp.study lesson "The Computational Steps of Standard
 * Self-Attention" and on the anylearn.cc page "Attention Is Memory-Bound, and
 * Nobody Noticed for Five Years". attn_fwd computes it as one fused tiled
 * kernel that never writes the N x N score or probability matrix to HBM
 * (pratikdhanave.com, "The Attention Bottleneck - and How FlashAttention Fixed
 * It", section "The fix: tiling and fusion, never touch HBM"); attn_fwd_naive
 * computes the same function as three separate kernels that materialise S and
 * P in HBM (the "standard path" of the anylearn.cc page).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Pointers q, k, v, o, lse, workspace are DEVICE pointers owned by the
 *   caller. The library never allocates or frees device memory, never
 *   synchronises the stream, and keeps no per-call state, so calls on
 *   different streams are independent.
 * - q, k, v, o: bf16 (IEEE binary16-brain, 2 bytes), layout [B, H, N, d]
 *   contiguous, i.e. element (b, h, i, c) at ((b*H + h)*N + i)*d + c. Must be
 *   16-byte aligned.
 * - lse: fp32 [B, H, N] contiguous, 4-byte aligned. lse[b,h,i] is the natural
 *   logarithm of sum_j exp(scale * q_i . k_j) over the allowed keys j.
 * - d (head dimension) must be 64 or 128 (the page's "d is 64 or 128").
 * - B, H, N >= 1; B*H*N must fit in a signed 32-bit int.
 * - scale: the logit multiplier (1/sqrt(d) for standard attention), applied
 *   as given; any finite value. scale = 0 gives the uniform softmax over the
 *   allowed keys (o = their mean of v, lse = ln of their count); a negative
 *   scale weights the keys with the lowest q . k highest. Non-finite scale:
 *   ATTN_ERR_SCALE.
 * - causal: 0 (every key) or 1 (key j allowed for query i iff j <= i).
 * - Arithmetic: bf16 operands, fp32 accumulation, fp32 softmax; O is rounded
 *   to bf16 (round to nearest even).
 * - Return value: ATTN_OK (0) or a negative ATTN_ERR_* code. On an argument
 *   error nothing is launched. A kernel that launched fine but failed on the
 *   device (the bounded-wait watchdog fired) is reported by
 *   attn_last_device_error().
 * - Asynchrony: work is enqueued on `stream` (a cudaStream_t; 0 = legacy
 *   default stream) and completes in stream order; errors of the kernel
 *   itself surface at the caller's next synchronisation.
 * - Device: an sm_100 (B200-class) device must be current; otherwise
 *   ATTN_ERR_UNSUPPORTED_DEVICE.
 */
#ifndef ATTN_B200_H
#define ATTN_B200_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *attn_stream_t; /* same type as cudaStream_t */

enum {
    ATTN_OK = 0,
    ATTN_ERR_NULL = -1,               /* a required pointer is NULL */
    ATTN_ERR_SHAPE = -2,              /* B, H or N < 1, or B*H*N too large */
    ATTN_ERR_HEADDIM = -3,            /* d is not 64 or 128 */
    ATTN_ERR_ALIGN = -4,              /* a pointer breaks its alignment rule */
    ATTN_ERR_SCALE = -5,              /* scale not finite; FP8 descale not finite and > 0 */
    ATTN_ERR_CAUSAL = -6,             /* causal is not 0 or 1 */
    ATTN_ERR_WORKSPACE = -7,          /* naive path: workspace too small */
    ATTN_ERR_LAUNCH = -8,             /* the CUDA launch failed */
    ATTN_ERR_UNSUPPORTED_DEVICE = -9, /* current device is not sm_100 */
    ATTN_ERR_TIMEOUT = -10,           /* a kernel gave up on a bounded wait */
    ATTN_ERR_CUDA = -11,              /* another CUDA runtime/driver call failed */
    ATTN_ERR_WINDOW = -12             /* attn_fwd_ext: a window bound below -1 */
};

/*
 * attn_fwd - fused exact attention forward (the hot path).
 *
 * One persistent-style grid of warp-specialised CTAs: TMA loads Q, K, V tiles
 * into swizzled shared memory through an mbarrier ring, tcgen05 MMAs
 * accumulate S = Q K^T and O += P V in tensor memory, and softmax warps keep a
 * running row maximum and row sum (online softmax, exp2 domain). S and P never
 * leave the SM; only O and lse are written. Each CTA works on 256 query rows
 * at a time; when B*H*ceil(N/256) is at most half the device's SMs, each CTA
 * takes 128 query rows instead and its two softmax groups split the keys
 * between them, merging their results at the end (twice the CTAs, no extra
 * memory). The two layouts agree within floating-point rounding, not bit
 * for bit.
 *
 * q, k, v (in), o (out): [B, H, N, d] bf16. lse (out): [B, H, N] fp32.
 * Returns ATTN_OK or ATTN_ERR_*; see the conventions above.
 */
int attn_fwd(const void *q, const void *k, const void *v, void *o, float *lse,
             int B, int H, int N, int d, float scale, int causal,
             attn_stream_t stream);

/*
 * attn_fwd_fp8 - attn_fwd with 8-bit floating-point inputs, the low-precision
 * step the anylearn.cc page credits FlashAttention-3 with (1.3 PFLOP/s in
 * FP8 on an H100). q, k, v hold OCP E4M3 codes (1 byte each, the finite-only
 * variant, largest value 448), [B, H, N, d] contiguous, 16-byte aligned; the
 * values attended are q_descale * Q, k_descale * K and v_descale * V (per-
 * tensor scales, finite and > 0, else ATTN_ERR_SCALE). d must be 128
 * (ATTN_ERR_HEADDIM). o: bf16 [B, H, N, d]; lse: fp32 [B, H, N], as for
 * attn_fwd. Both products run on the tensor cores in E4M3 with fp32
 * accumulation: S = Q K^T from the E4M3 inputs, and P (the softmax weights
 * 2^(x - m) <= 2^8, rounded to E4M3 to nearest) times V. The row sums and
 * the log-sum-exp use the unrounded fp32 weights.
 */
int attn_fwd_fp8(const void *q, const void *k, const void *v, void *o,
                 float *lse, int B, int H, int N, int d, float scale,
                 float q_descale, float k_descale, float v_descale, int causal,
                 attn_stream_t stream);

/*
 * attn_fwd_kv - fused attention of Nq query rows against Nk keys per head, the
 * long-context inference shape (a few new tokens against a long context:
 * pratikdhanave.com, "The Attention Bottleneck - and How FlashAttention Fixed
 * It", "Key takeaways", on context grown from 2K to 128K tokens). The article
 * describes no split of the key range; splitting it across CTAs and merging by
 * log-sum-exp is this library's reading of how to keep every SM busy when
 * B*H*ceil(Nq/128) CTAs cannot fill the GPU.
 *
 * q (in): [B, H, Nq, d] bf16. k, v (in): [B, H, Nk, d] bf16.
 * o (out): [B, H, Nq, d] bf16. lse (out): [B, H, Nq] fp32.
 * Causal alignment is bottom-right: query row i is sequence position
 * i + (Nk - Nq), and sees key j iff j <= i + (Nk - Nq) (so Nq == Nk is the
 * square causal problem of attn_fwd, and Nq = 1 sees every key). Causal needs
 * Nq <= Nk (ATTN_ERR_SHAPE otherwise).
 *
 * The keys are cut into 128-key tiles and the tiles into num_splits ranges of
 * equal length (the last may be shorter; a request above the tile count is
 * clamped to it, and a count that would leave a range empty is lowered). Each
 * (head, query block, range) is one CTA of the fused kernel, which writes a
 * normalised fp32 partial O and its lse per range; a second kernel combines
 * them, O = sum_s w_s O_s / sum_s w_s with w_s = exp(lse_s - max_s lse_s).
 * With num_splits = 1 the fused kernel writes o and lse directly; when also
 * Nq == Nk the call runs what attn_fwd runs for that shape (for
 * attn_fwd_ext, with its window and bias), with the same results as attn_fwd
 * where no window or bias is asked for.
 *
 * num_splits: 1 .. 256, or 0 for attn_fwd_kv_num_splits(...)'s choice.
 * workspace: device memory of at least
 * attn_fwd_kv_workspace_bytes(B, H, Nq, Nk, d, num_splits) bytes, 256-byte
 * aligned; NULL is allowed when that is 0. Other conventions as for attn_fwd
 * (B, H, Nq, Nk >= 1; B*H*Nq and B*H*Nk fit in a signed 32-bit int).
 */
int attn_fwd_kv(const void *q, const void *k, const void *v, void *o,
                float *lse, int B, int H, int Nq, int Nk, int d, float scale,
                int causal, int num_splits, void *workspace,
                size_t workspace_bytes, attn_stream_t stream);

/*
 * attn_fwd_kv_num_splits - the split count attn_fwd_kv uses for num_splits = 0
 * on the current device: 1 when B*H*ceil(Nq/rows) CTAs already fill the SMs
 * (rows = 128 for Nq <= 128, else 256), otherwise the fewest splits whose
 * waves of CTAs are within 15% of the best SM utilisation, with at least 8 KV
 * tiles per split. Returns a count >= 1, or a negative ATTN_ERR_* code.
 */
int attn_fwd_kv_num_splits(int B, int H, int Nq, int Nk, int d);

/*
 * attn_fwd_kv_workspace_bytes - workspace attn_fwd_kv needs for this shape and
 * num_splits (0 = the automatic choice on the current device): with s > 1
 * effective splits, s*B*H*Nq*d fp32 partial outputs (rounded up to 256 bytes)
 * followed by s*B*H*Nq fp32 partial lse values; 0 when s = 1 or the arguments
 * are invalid.
 */
size_t attn_fwd_kv_workspace_bytes(int B, int H, int Nq, int Nk, int d,
                                   int num_splits);

/*
 * attn_fwd_ext - attn_fwd_kv with the variants a fused library usually does
 * not cover (the anylearn.cc page "Attention Is Memory-Bound, and Nobody
 * Noticed for Five Years", on why the library matters, names bespoke biases,
 * masks and position encodings as what leaves the fast path), computed inside
 * the same fused kernel:
 *
 * - a key window around the query's sequence position pos = i + (Nk - Nq):
 *   key j is allowed iff pos - window_left <= j (when window_left >= 0) and
 *   j <= pos + window_right (when window_right >= 0), on top of the causal
 *   rule; -1 leaves that side unbounded. causal = 1 with window_left = W - 1
 *   is a sliding window of the W most recent keys. KV tiles wholly outside
 *   every row's window are never loaded.
 * - alibi_slopes: NULL, or H device floats (4-byte aligned, finite); the
 *   logit of key j for a query at position pos becomes
 *   scale * q.k_j - alibi_slopes[h] * |pos - j| (a per-head linear distance
 *   bias; natural-log units, added after the scale).
 *
 * A row with no allowed key gets O = 0 and lse = -inf. Other arguments,
 * layouts and the split / workspace rules as for attn_fwd_kv, except that the
 * splits cut only the key tiles from the first row's window start on; size
 * the workspace with attn_fwd_ext_workspace_bytes. ATTN_ERR_WINDOW if a
 * window bound is below -1.
 */
int attn_fwd_ext(const void *q, const void *k, const void *v, void *o,
                 float *lse, int B, int H, int Nq, int Nk, int d, float scale,
                 int causal, int window_left, int window_right,
                 const float *alibi_slopes, int num_splits, void *workspace,
                 size_t workspace_bytes, attn_stream_t stream);

/* attn_fwd_ext_num_splits - the automatic split count of attn_fwd_ext on the
 * current device (>= 1), or a negative ATTN_ERR_* code. */
int attn_fwd_ext_num_splits(int B, int H, int Nq, int Nk, int d, int window_left);

/* attn_fwd_ext_workspace_bytes - workspace attn_fwd_ext needs for num_splits
 * (0 = automatic on the current device); 0 when one split or invalid. */
size_t attn_fwd_ext_workspace_bytes(int B, int H, int Nq, int Nk, int d,
                                    int window_left, int num_splits);

/*
 * attn_fwd_naive_workspace_bytes - bytes of workspace attn_fwd_naive needs:
 * 2 * (B*H*N*N) bf16 values (S, then P), i.e. 4*B*H*N*N bytes. Returns 0 if
 * the arguments are not positive or the size overflows.
 */
size_t attn_fwd_naive_workspace_bytes(int B, int H, int N);

/*
 * attn_fwd_naive - the deliberately unfused standard path: three kernels on
 * `stream`,
 *   1. S = scale * Q K^T   (causally masked entries set to -inf), bf16, to HBM
 *   2. P = softmax(S) row-wise, bf16, to HBM; lse in fp32
 *   3. O = P V, bf16
 * so each N x N matrix crosses the HBM boundary twice (four crossings in all,
 * as the anylearn.cc page counts them). Same arguments and result as
 * attn_fwd, plus a caller-owned device workspace of at least
 * attn_fwd_naive_workspace_bytes(B, H, N) bytes, 16-byte aligned (S at offset
 * 0, P right after it). Extra limits: N <= 32768 and B*H <= 65535
 * (ATTN_ERR_SHAPE otherwise). A smaller workspace returns ATTN_ERR_WORKSPACE.
 */
int attn_fwd_naive(const void *q, const void *k, const void *v, void *o,
                   float *lse, int B, int H, int N, int d, float scale,
                   int causal, void *workspace, size_t workspace_bytes,
                   attn_stream_t stream);

/*
 * ATTN_NOALLOC_SCRATCH_BYTES - size of the fixed device scratch array behind
 * attn_fwd_naive_noalloc (64 MiB). Every GPU that loads the library holds it
 * until the process exits.
 */
#define ATTN_NOALLOC_SCRATCH_BYTES (64u * 1024u * 1024u)

/*
 * attn_fwd_naive_noalloc - attn_fwd_naive for callers that must not allocate
 * device memory. The pages describe no such entry point: it has no
 * counterpart there. It exists for callers that cannot call cudaMalloc or
 * hand over a workspace: code embedded in a host framework that owns the
 * whole device-memory budget through its own pool and forbids allocations
 * outside it, and latency-bound loops where cudaMalloc/cudaFree would add
 * their implicit device-wide synchronisation.
 *
 * Same arguments, limits and result as attn_fwd_naive, minus the workspace:
 * S and P go to a library-owned device array of ATTN_NOALLOC_SCRATCH_BYTES,
 * so 4*B*H*N*N must not exceed it (ATTN_ERR_WORKSPACE otherwise, before any
 * launch). The function allocates nothing itself: no cudaMalloc, cudaFree or
 * allocating library call.
 *
 * - Set-up: the first call on each device looks up the array's device address
 *   (cudaGetSymbolAddress, with that device current) and caches it; make that
 *   first call before any stream capture on that device.
 * - Sharing: every call on a device uses the same array, which keeps the
 *   previous call's contents. The three kernels overwrite every element of S
 *   and P they read, so nothing has to start at zero. Calls whose work
 *   overlaps on the GPU (different streams without ordering between them)
 *   race on the array and give wrong results; order them on one stream.
 */
int attn_fwd_naive_noalloc(const void *q, const void *k, const void *v,
                           void *o, float *lse, int B, int H, int N, int d,
                           float scale, int causal, attn_stream_t stream);

/*
 * attn_last_device_error - reads and clears the device-side error word of the
 * current device. Every wait inside the fused kernel is bounded; a CTA whose
 * wait runs out sets this word, drains its own copies, frees its tensor memory
 * and exits. Returns ATTN_OK, ATTN_ERR_TIMEOUT, or ATTN_ERR_CUDA if the query
 * itself failed. Synchronises `stream` (the only entry point that does).
 */
int attn_last_device_error(attn_stream_t stream);

/*
 * attn_set_wait_limit_ms - sets the limit, in milliseconds of the device's
 * global timer, of every bounded wait inside the library's kernels, for
 * launches made after the call (process-wide; default 2000). A wait that runs
 * out makes its CTA give up as described under attn_last_device_error. Raise
 * it where the GPU is time-sliced with other work for long stretches, so that
 * a preempted CTA is not mistaken for a stuck one; lower it to fail faster.
 * ms: 1 .. 600000, else ATTN_ERR_SHAPE. attn_wait_limit_ms returns the value
 * in effect.
 */
int attn_set_wait_limit_ms(int ms);
int attn_wait_limit_ms(void);

/* attn_status_string - a static, human-readable name for a status code. */
const char *attn_status_string(int status);

/*
 * attn_selftest_wait_timeout - watchdog check. Launches one CTA that waits, with
 * the same bounded wait the fused kernel uses, on an mbarrier nothing ever
 * arrives on, with a limit of `limit_ms` milliseconds (1..5000). The kernel then
 * records the timeout and returns; the device stays usable. After a stream
 * synchronisation attn_last_device_error() must report ATTN_ERR_TIMEOUT.
 */
int attn_selftest_wait_timeout(int limit_ms, attn_stream_t stream);

/*
 * attn_selftest_exp2 - numerics check of the exponential the fused kernel
 * evaluates on the FMA pipe for part of each softmax row (the rest uses the
 * MUFU's ex2): 2^x by Cody-Waite range reduction (x = j + f, |f| <= 1/2) and a
 * minimax cubic for 2^f, with j added to the exponent field; inputs below -125
 * give a tiny positive value (<= 2^-124) in place of 0. x, y: n device floats,
 * 4-byte aligned; y[i] = 2^x[i]. Launches one kernel on `stream`.
 */
int attn_selftest_exp2(const float *x, float *y, int n, attn_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* ATTN_B200_H */
