"""Seeded synthetic inputs and row samples, shared by the tests, the smoke check
and the benchmark.

This module holds no attention arithmetic: it only draws Q, K, V and chooses
which query rows a large-shape check compares. Both the CUDA path and the
oracle receive the very same bf16 tensors produced here.

Workloads (the five shapes the method is measured on):

* ``single_head_128``        B=1,  H=1,  N=128,   d=64,  non-causal, Q,K,V ~ N(0,1)
* ``bert_base_1024``         B=1,  H=12, N=1024,  d=64,  non-causal, Q,K,V ~ N(0,1)
* ``decoder_2048_causal``    B=8,  H=32, N=2048,  d=128, causal,     Q,K,V ~ N(0,1)
* ``long_8192_causal``       B=8,  H=32, N=8192,  d=128, causal,     Q,K,V ~ N(0,1)
  (the batch/head/length of the score-matrix memory example on the anylearn.cc
  page "Attention Is Memory-Bound, and Nobody Noticed for Five Years")
* ``stress_65536_causal``    B=1,  H=32, N=65536, d=128, causal,     Q,K ~ N(0,4^2), V ~ U(-1,1)

Inference shapes (Nq query rows against Nk keys, causal alignment bottom-right):

* ``decode_131072``            B=4, H=32, Nq=1,   Nk=131072, d=128, Q,K,V ~ N(0,1)
  (one new token per sequence against a 128K-token context, the upper end of
  the 2K to 128K context growth on the pratikdhanave.com article "The
  Attention Bottleneck - and How FlashAttention Fixed It", "Key takeaways")
* ``decode_32768``             B=4, H=32, Nq=1,   Nk=32768,  d=128 (the same at a
  quarter of the context: small enough for multi-pass profiler captures)
* ``chunk_128x32768_causal``   B=4, H=32, Nq=128, Nk=32768,  d=128, causal
* ``chunk_512x8192_causal``    B=2, H=16, Nq=512, Nk=8192,   d=128, causal

Draws are fp32 from a CPU ``torch.Generator`` seeded with the given seed, in the
order Q, K, V, then rounded to bf16 (round to nearest even).
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np
import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    N: int
    d: int
    causal: bool
    dist: str  # "normal" or "stress"
    seed: int
    sampled: bool  # True: check a seeded row sample; False: every row

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    @property
    def shape(self):
        return (self.B, self.H, self.N, self.d)


WORKLOADS = {
    w.name: w
    for w in (
        Workload("single_head_128", 1, 1, 128, 64, False, "normal", 1001, False),
        Workload("bert_base_1024", 1, 12, 1024, 64, False, "normal", 1002, False),
        Workload("decoder_2048_causal", 8, 32, 2048, 128, True, "normal", 1003, True),
        Workload("long_8192_causal", 8, 32, 8192, 128, True, "normal", 1004, True),
        Workload("stress_65536_causal", 1, 32, 65536, 128, True, "stress", 1005, True),
    )
}


@dataclass(frozen=True)
class KvWorkload:
    name: str
    B: int
    H: int
    Nq: int
    Nk: int
    d: int
    causal: bool
    dist: str
    seed: int
    rows_per_head: int  # query rows per (b, h) the parity check compares (all if >= Nq)

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)


KV_WORKLOADS = {
    w.name: w
    for w in (
        KvWorkload("decode_131072", 4, 32, 1, 131072, 128, False, "normal", 1101, 1),
        KvWorkload("decode_32768", 4, 32, 1, 32768, 128, False, "normal", 1104, 1),
        KvWorkload("chunk_128x32768_causal", 4, 32, 128, 32768, 128, True, "normal", 1102, 16),
        KvWorkload("chunk_512x8192_causal", 2, 16, 512, 8192, 128, True, "normal", 1103, 32),
    )
}


def _draw(g, shape, dist):
    if dist == "normal":
        return torch.randn(shape, generator=g, dtype=torch.float32)
    if dist == "grid8":
        return torch.randint(-32, 33, shape, generator=g).to(torch.float32) / 8.0
    raise ValueError(f"unknown distribution {dist!r}")


def make_q_kv(B: int, H: int, Nq: int, Nk: int, d: int, seed: int, dist: str = "normal"):
    """Q [B, H, Nq, d] and K, V [B, H, Nk, d] as contiguous CPU bf16 tensors,
    drawn in the order Q, K, V ("normal" or "grid8" as in make_qkv)."""
    g = torch.Generator(device="cpu").manual_seed(int(seed))
    q = _draw(g, (B, H, Nq, d), dist)
    k = _draw(g, (B, H, Nk, d), dist)
    v = _draw(g, (B, H, Nk, d), dist)
    return (q.to(torch.bfloat16), k.to(torch.bfloat16), v.to(torch.bfloat16))


def make_kv_workload(w: KvWorkload):
    return make_q_kv(w.B, w.H, w.Nq, w.Nk, w.d, w.seed, w.dist)


def make_qkv(B: int, H: int, N: int, d: int, seed: int, dist: str = "normal"):
    """Q, K, V as contiguous CPU torch.bfloat16 tensors of shape [B, H, N, d]."""
    g = torch.Generator(device="cpu").manual_seed(int(seed))
    shape = (B, H, N, d)
    if dist == "normal":
        q = torch.randn(shape, generator=g, dtype=torch.float32)
        k = torch.randn(shape, generator=g, dtype=torch.float32)
        v = torch.randn(shape, generator=g, dtype=torch.float32)
    elif dist == "stress":
        q = torch.randn(shape, generator=g, dtype=torch.float32).mul_(4.0)
        k = torch.randn(shape, generator=g, dtype=torch.float32).mul_(4.0)
        v = torch.rand(shape, generator=g, dtype=torch.float32).mul_(2.0).sub_(1.0)
    elif dist == "grid8":
        # multiples of 1/8 in [-4, 4]: exactly representable in bf16, and so is
        # the sum of two of them (|x| <= 8, step 1/8).
        def grid():
            return torch.randint(-32, 33, shape, generator=g).to(torch.float32) / 8.0
        q, k, v = grid(), grid(), grid()
    else:
        raise ValueError(f"unknown distribution {dist!r}")
    return (q.to(torch.bfloat16), k.to(torch.bfloat16), v.to(torch.bfloat16))


def make_workload(w: Workload):
    return make_qkv(w.B, w.H, w.N, w.d, w.seed, w.dist)


_MASK64 = (1 << 64) - 1


def splitmix64(state: int):
    """One step of SplitMix64 (Steele, Lea and Flood, 2014). Returns (value, state)."""
    state = (state + 0x9E3779B97F4A7C15) & _MASK64
    z = state
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _MASK64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _MASK64
    return z ^ (z >> 31), state


def sample_rows(seed: int, BH: int, N: int, per_head: int = 256) -> np.ndarray:
    """Seeded (bh, i) pairs: per head the rows 0 and N-1 plus distinct rows
    drawn from a SplitMix64 stream seeded with seed ^ bh, sorted; every row
    when N <= per_head. Returns int64 [R, 2]."""
    out = []
    for bh in range(BH):
        if N <= per_head:
            rows = list(range(N))
        else:
            chosen = {0, N - 1}
            state = (int(seed) ^ bh) & _MASK64
            while len(chosen) < per_head:
                z, state = splitmix64(state)
                chosen.add(int(z % N))
            rows = sorted(chosen)
        out.extend((bh, i) for i in rows)
    return np.asarray(out, dtype=np.int64).reshape(-1, 2)


def gather_rows(t: torch.Tensor, rows: np.ndarray) -> torch.Tensor:
    """Rows of a [B, H, N, ...] tensor at (bh, i) pairs -> [R, ...]."""
    B, H, N = t.shape[:3]
    flat = t.reshape(B * H * N, *t.shape[3:])
    idx = torch.as_tensor(rows[:, 0] * N + rows[:, 1], dtype=torch.long, device=t.device)
    return flat.index_select(0, idx)


def quantize_e4m3(t: torch.Tensor, target_amax: float = 448.0):
    """Per-tensor E4M3 quantisation of a float tensor (any device): returns
    (codes as torch.float8_e4m3fn, descale) with t ~= descale * codes; the
    scale maps the tensor's largest magnitude to target_amax (round to
    nearest, saturating)."""
    amax = float(t.detach().abs().max().float().cpu())
    descale = (amax / target_amax) if amax > 0 else 1.0
    codes = (t.float() / descale).clamp(-448.0, 448.0).to(torch.float8_e4m3fn)
    return codes, descale


def make_qkv_fp8(B: int, H: int, N: int, d: int, seed: int):
    """make_qkv's N(0,1) draws, quantised per tensor to E4M3: returns
    ((q8, k8, v8), (q_descale, k_descale, v_descale)) on the CPU."""
    q, k, v = make_qkv(B, H, N, d, seed)
    out = [quantize_e4m3(x) for x in (q, k, v)]
    return tuple(c for c, _ in out), tuple(s for _, s in out)
