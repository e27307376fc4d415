/*
 * chain.h - the elementwise-chain example, fused and unfused
 * (part of libattn_b200.so).
 *
 * The anylearn.cc page "Attention Is Memory-Bound, and Nobody Noticed for
 * Five Years" (the paragraphs on the technique underneath) gives the small
 * case of the fusion principle the attention kernel applies: a chain of a
 * scaling, a bias and an activation. Run as three kernels, it reads and
 * writes the whole tensor three times; one fused kernel reads it once and
 * writes the result once, the intermediates staying in registers, and should
 * run about three times faster because the arithmetic was never the cost.
 *
 * Operation, for x [rows, cols] and a per-column bias b [cols]:
 *
 *     y[r, c] = act(alpha * x[r, c] + b[c])
 *
 * act: CHAIN_ACT_RELU max(z, 0); CHAIN_ACT_GELU z * Phi(z) with the exact
 * normal CDF Phi(z) = (1 + erf(z / sqrt 2)) / 2; CHAIN_ACT_SILU z / (1 + e^-z);
 * CHAIN_ACT_GELU_TANH z (1 + tanh(sqrt(2/pi) (z + 0.044715 z^3))) / 2, the
 * tanh form of GELU that GPT-2 uses.
 *
 * Conventions: x, b, y, tmp are bf16 DEVICE pointers owned by the caller,
 * 16-byte aligned, row-major contiguous; cols must be a multiple of 8 and
 * rows * cols must fit in a signed 64-bit count (rows, cols >= 1). alpha must
 * be finite. Work is enqueued on `stream`; nothing is allocated or
 * synchronised. Return values are the ATTN_* codes of attn.h: ATTN_ERR_NULL,
 * ATTN_ERR_SHAPE (sizes, or cols not a multiple of 8), ATTN_ERR_ALIGN,
 * ATTN_ERR_SCALE (alpha not finite), ATTN_ERR_CAUSAL (act out of range),
 * ATTN_ERR_UNSUPPORTED_DEVICE, ATTN_ERR_LAUNCH.
 */
#ifndef CHAIN_B200_H
#define CHAIN_B200_H

#include <stddef.h>

#include "attn.h"

#ifdef __cplusplus
extern "C" {
#endif

enum { CHAIN_ACT_RELU = 0, CHAIN_ACT_GELU = 1, CHAIN_ACT_SILU = 2, CHAIN_ACT_GELU_TANH = 3 };

/*
 * chain_fused - one kernel: reads x (and b), computes alpha * x + b and the
 * activation in fp32 registers, writes y rounded to bf16 (nearest even).
 */
int chain_fused(const void *x, const void *b, void *y, long long rows, int cols,
                float alpha, int act, attn_stream_t stream);

/*
 * chain_unfused - the same chain as three kernels, each a full pass over the
 * tensor through HBM with its result rounded to bf16: tmp = alpha * x;
 * tmp = tmp + b (in place); y = act(tmp). tmp: caller-owned [rows, cols]
 * bf16 scratch (16-byte aligned), distinct from x and y.
 */
int chain_unfused(const void *x, const void *b, void *y, void *tmp, long long rows,
                  int cols, float alpha, int act, attn_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* CHAIN_B200_H */
