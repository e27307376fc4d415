"""FLOP and HBM-byte models used for the throughput and roofline figures.

* FLOPs: two matrix products of 2*N*N*d multiply-adds each per head, so
  4*B*H*N^2*d, halved when causal (only the lower triangle is useful work).
* Fused bytes: the fused path reads Q, K, V once and writes O once (bf16) and
  the fp32 log-sum-exp, so 8*B*H*N*d + 4*B*H*N ("You pay the HBM cost once
  (read inputs, write output)": pratikdhanave.com, "The Attention Bottleneck -
  and How FlashAttention Fixed It", section "The fix: tiling and fusion").
* Naive bytes: the N x N score matrix S and probability matrix P, each 16-bit,
  cross the HBM boundary four times in all (S written, S read, P written,
  P read) as traced on the anylearn.cc page "Attention Is Memory-Bound, and
  Nobody Noticed for Five Years"; on top of that Q, K, V are read and O and
  the log-sum-exp are written once.
* Inference shapes (Nq query rows against Nk keys, causal alignment
  bottom-right): query i sees min(Nk, i + Nk - Nq + 1) keys when causal, all
  Nk otherwise; FLOPs are 4*d per (query, visible key) pair. The fused kernel
  reads Q, K, V once and writes O and lse once: 2*B*H*(2*Nq + 2*Nk)*d + 4*B*H*Nq
  bytes (the split partials and their combine are overhead, not algorithmic).
"""
from __future__ import annotations


def attn_flops(B: int, H: int, N: int, d: int, causal: bool) -> float:
    f = 4.0 * B * H * N * N * d
    return f / 2.0 if causal else f


def score_matrix_bytes(N: int, heads: int = 1, batch: int = 1, elem_bytes: int = 2) -> int:
    """Bytes of one materialised N x N matrix per (batch, head), summed."""
    return elem_bytes * batch * heads * N * N


def score_crossings_bytes(N: int, heads: int = 1, batch: int = 1, elem_bytes: int = 2) -> int:
    """The four HBM crossings of the N x N intermediates (S out, S in, P out, P in)."""
    return 4 * score_matrix_bytes(N, heads, batch, elem_bytes)


def fused_bytes(B: int, H: int, N: int, d: int) -> int:
    return 8 * B * H * N * d + 4 * B * H * N


def naive_bytes(B: int, H: int, N: int, d: int) -> int:
    return score_crossings_bytes(N, H, B) + 8 * B * H * N * d + 4 * B * H * N


def naive_kernel_bytes(B: int, H: int, N: int, d: int) -> dict:
    """Algorithmic bytes of each of the three unfused kernels."""
    bhn, s = B * H * N, score_matrix_bytes(N, H, B)
    return {
        "scores": 4 * bhn * d + s,          # read Q, K; write S
        "softmax": 2 * s + 4 * bhn,         # read S; write P and lse
        "values": s + 4 * bhn * d,          # read P, V; write O
    }


def traffic_seconds(nbytes: float, bytes_per_s: float) -> float:
    return nbytes / bytes_per_s


def tile_pairs(B: int, H: int, N: int, causal: bool, tile: int = 128) -> int:
    """(query tile, key tile) pairs a tiled kernel visits with causal skipping."""
    t = -(-N // tile)
    per_head = t * (t + 1) // 2 if causal else t * t
    return B * H * per_head


def kv_visible_pairs(Nq: int, Nk: int, causal: bool) -> int:
    """(query, key) pairs with the key visible, per head."""
    if not causal:
        return Nq * Nk
    if Nq > Nk:
        raise ValueError("causal needs Nq <= Nk")
    # query i sees i + (Nk - Nq) + 1 <= Nk keys
    return Nq * (Nk - Nq + 1) + Nq * (Nq - 1) // 2


def kv_flops(B: int, H: int, Nq: int, Nk: int, d: int, causal: bool) -> float:
    return 4.0 * B * H * d * kv_visible_pairs(Nq, Nk, causal)


def kv_bytes(B: int, H: int, Nq: int, Nk: int, d: int) -> int:
    return 2 * B * H * (2 * Nq + 2 * Nk) * d + 4 * B * H * Nq


def ext_visible_pairs(Nq: int, Nk: int, causal: bool, window_left: int = -1,
                      window_right: int = -1) -> int:
    """(query, key) pairs allowed by the causal rule and a key window
    [pos - window_left, pos + window_right] around pos = i + Nk - Nq, per head."""
    total = 0
    off = Nk - Nq
    for i in range(Nq):
        pos = i + off
        hi = Nk - 1
        if causal:
            hi = min(hi, pos)
        if window_right >= 0:
            hi = min(hi, pos + window_right)
        lo = max(0, pos - window_left) if window_left >= 0 else 0
        total += max(0, hi - lo + 1)
    return total
