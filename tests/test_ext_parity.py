"""attn_fwd_ext (key windows around the query position and a per-head linear
distance bias, inside the fused kernel) against the fp64 oracle, element by
element on every row. Covers sliding windows (causal with a left bound),
two-sided windows without the causal rule, a window of one key, the distance
bias alone and together with a window, decode and prefill shapes, both CTA
layouts, explicit and automatic split counts, and rows with no allowed key
(O = 0, lse = -inf on both sides).
"""
import numpy as np
import pytest
import torch

import exact_attention_125_b200 as ea
import oracle
from exact_attention_125_b200.inputs import gather_rows, make_q_kv, sample_rows
from parity_util import assert_within, compare, scale_of

pytestmark = pytest.mark.gpu

CASES = [
    # B, H, Nq, Nk, d, causal, window_left, window_right, slopes, num_splits
    (1, 2, 300, 300, 128, True, 63, -1, None, 1),
    (1, 2, 300, 300, 64, True, 200, -1, "alibi", 1),
    (2, 2, 1, 5000, 128, True, 1000, -1, None, 0),
    (1, 4, 1, 3000, 128, False, -1, -1, "alibi", 3),
    (1, 2, 100, 1100, 128, True, 300, -1, "steep", 4),
    (1, 2, 129, 700, 64, False, 100, 50, None, 2),
    (1, 1, 600, 600, 128, False, 0, 0, None, 1),
    (1, 2, 256, 256, 128, True, -1, -1, "alibi", 1),
    (1, 2, 500, 2000, 128, True, 127, -1, None, 5),
    (1, 2, 700, 700, 128, True, 255, -1, "steep", 0),
    (1, 1, 300, 200, 64, False, 10, 10, None, 1),   # early rows: no key in their window
    (1, 3, 17, 4096, 64, True, 511, -1, "alibi", 0),
    # Square problems with one split: with few heads (at most half as many
    # 256-row units as SMs) they run one 128-row query tile per CTA on the kv
    # kernel; with many heads (*_SQ below) on the persistent square kernel's
    # window and bias instantiations. Non-causal (tiles left of, right of and
    # across the diagonal), steep slopes (the bias added per logit, or a
    # bound up to the slack above the row maximum), one-sided and two-sided
    # windows, a window wider than N, the diagonal alone, ragged N, both head
    # sizes.
    (1, 2, 300, 300, 128, False, -1, -1, "alibi", 1),
    (1, 2, 513, 513, 64, True, -1, -1, "steep", 0),
    (2, 2, 384, 384, 128, False, -1, -1, "steep", 1),
    (2, 40, 700, 700, 128, True, 200, -1, None, 1),
    (1, 160, 520, 520, 64, True, 300, -1, "alibi", 1),
    (1, 3, 1000, 1000, 64, False, 100, 300, None, 1),
    (1, 2, 900, 900, 128, False, 250, 250, "steep", 1),
    (1, 2, 513, 513, 128, True, 5000, 3, "alibi", 1),
    (1, 2, 640, 640, 128, False, 129, -1, None, 1),
    (1, 2, 640, 640, 64, False, -1, 129, "alibi", 1),
    (1, 2, 384, 384, 128, True, 0, -1, None, 1),
    # the same square window problem cut into key-range splits (kv path)
    (1, 2, 300, 300, 128, True, 63, -1, None, 2),
    (1, 3, 513, 513, 128, True, -1, -1, "steep", 1),
    (1, 2, 777, 777, 64, True, -1, -1, "alibi", 1),
    (1, 2, 640, 640, 128, True, 200, -1, "steep", 1),
]

# Many heads: the persistent square kernel's window and bias instantiations
# (more 256-row units than half the SMs; several per CTA where they
# outnumber the SMs).
CASES_SQ = [
    (1, 40, 300, 300, 128, False, -1, -1, "alibi", 1),
    (1, 40, 384, 384, 128, False, -1, -1, "steep", 1),
    (1, 40, 1000, 1000, 64, False, 100, 300, None, 1),
    (1, 40, 900, 900, 128, False, 250, 250, "steep", 1),
    (1, 40, 513, 513, 128, True, 5000, 3, "alibi", 1),
    (1, 30, 640, 640, 128, False, 129, -1, None, 1),
    (1, 30, 640, 640, 64, False, -1, 129, "alibi", 1),
    (1, 60, 384, 384, 128, True, 0, -1, None, 1),
    (1, 40, 513, 513, 128, True, -1, -1, "steep", 1),
    (1, 40, 777, 777, 64, True, -1, -1, "alibi", 1),
    (1, 40, 640, 640, 128, True, 200, -1, "steep", 1),
]


def _slopes(kind, H):
    if kind is None:
        return None
    if kind == "alibi":  # the geometric slopes 2^(-8 (h + 1) / H)
        return [2.0 ** (-8.0 * (h + 1) / H) for h in range(H)]
    return [0.5 / (h + 1) for h in range(H)]  # steep: a few keys dominate


@pytest.mark.parametrize("B,H,Nq,Nk,d,causal,wl,wr,kind,splits", CASES + CASES_SQ)
def test_ext_all_rows(B, H, Nq, Nk, d, causal, wl, wr, kind, splits):
    _ext_case(B, H, Nq, Nk, d, causal, wl, wr, kind, splits, scale_of(d))


@pytest.mark.parametrize("scale", [0.0, -0.1])
@pytest.mark.parametrize("B,H,Nq,Nk,d,causal,wl,wr,kind,splits", [
    (1, 2, 300, 300, 128, True, 63, -1, "alibi", 1),
    (1, 2, 100, 1100, 128, True, 300, -1, None, 4),
    (1, 4, 1, 3000, 64, False, -1, -1, "alibi", 3),
    (1, 2, 300, 300, 128, True, -1, -1, "alibi", 1),
    (1, 40, 300, 300, 128, True, 63, -1, "alibi", 1),
    (1, 40, 300, 300, 128, False, -1, -1, "steep", 1),
])
def test_ext_zero_and_negative_scale(B, H, Nq, Nk, d, causal, wl, wr, kind, splits, scale):
    _ext_case(B, H, Nq, Nk, d, causal, wl, wr, kind, splits, scale)


def _ext_case(B, H, Nq, Nk, d, causal, wl, wr, kind, splits, scale):
    q, k, v = make_q_kv(B, H, Nq, Nk, d, seed=Nq * 13 + Nk + wl + 7 * wr + d)
    slopes = _slopes(kind, H)
    qg, kg, vg = (t.to("cuda") for t in (q, k, v))
    sl = torch.tensor(slopes, dtype=torch.float32, device="cuda") if slopes else None
    o = torch.full((B, H, Nq, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((B, H, Nq), float("nan"), dtype=torch.float32, device="cuda")
    ea.attn_fwd_ext(qg, kg, vg, o, lse, scale=scale, causal=causal, window_left=wl,
                    window_right=wr, alibi_slopes=sl, num_splits=splits)
    torch.cuda.synchronize()
    assert ea.last_device_error() == 0
    rows = oracle.all_rows(B * H, Nq)
    # the oracle gets the fp32 slopes the kernel uses, widened exactly
    sl64 = [float(np.float32(x)) for x in slopes] if slopes else None
    o_ref, lse_ref = oracle.attention_ext(q, k, v, scale, causal, wl, wr, sl64, rows=rows)
    o_rows = gather_rows(o.cpu(), rows)
    lse_rows = gather_rows(lse.cpu().unsqueeze(-1), rows).squeeze(-1)
    empty = np.isneginf(lse_ref)
    if empty.any():
        assert np.isneginf(lse_rows.numpy()[empty]).all()
        assert (o_rows.float().numpy()[empty] == 0).all()
    keep = ~empty
    e = compare(o_rows[torch.as_tensor(keep)], lse_rows[torch.as_tensor(keep)], o_ref[keep],
                lse_ref[keep])
    assert_within(e, f"{(B, H, Nq, Nk, d, causal, wl, wr, kind, splits, scale)}")


def test_ext_without_options_matches_attn_fwd_kv_bit_for_bit():
    q, k, v = make_q_kv(1, 2, 40, 3000, 128, seed=9)
    qg, kg, vg = (t.to("cuda") for t in (q, k, v))
    o1, l1 = ea.attn_fwd_kv(qg, kg, vg, causal=True, num_splits=3)
    o2, l2 = ea.attn_fwd_ext(qg, kg, vg, causal=True, num_splits=3)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


@pytest.mark.parametrize("H", [3, 40])  # the one-tile layout and the 256-row kernel
@pytest.mark.parametrize("causal", [False, True])
def test_square_ext_without_options_matches_attn_fwd_bit_for_bit(causal, H):
    # Nq == Nk, no window, no bias: both entry points take the same layout
    q, k, v = make_q_kv(1, H, 700, 700, 128, seed=11 + int(causal))
    qg, kg, vg = (t.to("cuda") for t in (q, k, v))
    o1, l1 = ea.attn_fwd(qg, kg, vg, causal=causal)
    o2, l2 = ea.attn_fwd_ext(qg, kg, vg, causal=causal, num_splits=1)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


@pytest.mark.parametrize("H", [3, 40])  # the one-tile layout and the 256-row kernel
@pytest.mark.parametrize("alibi", [False, True])
@pytest.mark.parametrize("causal", [False, True])
def test_square_window_over_every_key_matches_unwindowed_bit_for_bit(causal, alibi, H):
    # a window wider than the sequence masks nothing: the window
    # instantiation must then reproduce the unwindowed kernel exactly (same
    # tiles, same masks, same arithmetic order)
    N = 700
    q, k, v = make_q_kv(1, H, N, N, 128, seed=23 + int(causal) + 2 * int(alibi))
    qg, kg, vg = (t.to("cuda") for t in (q, k, v))
    sl = (torch.tensor([2.0 ** (-8.0 * (h + 1) / H) for h in range(H)], dtype=torch.float32,
                       device="cuda") if alibi else None)
    o1, l1 = ea.attn_fwd_ext(qg, kg, vg, causal=causal, alibi_slopes=sl, num_splits=1)
    o2, l2 = ea.attn_fwd_ext(qg, kg, vg, causal=causal, window_left=N, window_right=N,
                             alibi_slopes=sl, num_splits=1)
    torch.cuda.synchronize()
    assert ea.last_device_error() == 0
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


@pytest.mark.parametrize("B,H,N,wl,alibi", [
    # the benchmark's two shapes with fewer heads: a 4096-key sliding window
    # over a 32768-token causal prefill, and the distance bias at 8192 (the
    # slopes of the benchmark's 32 heads, first eight)
    (1, 4, 32768, 4095, False),
    (1, 8, 8192, -1, True),
])
def test_benchmark_shapes_sampled_rows(B, H, N, wl, alibi):
    d = 128
    q, k, v = make_q_kv(B, H, N, N, d, seed=N + wl + int(alibi))
    slopes = [2.0 ** (-8.0 * (h + 1) / 32) for h in range(H)] if alibi else None
    qg, kg, vg = (t.to("cuda") for t in (q, k, v))
    sl = torch.tensor(slopes, dtype=torch.float32, device="cuda") if slopes else None
    o = torch.full((B, H, N, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((B, H, N), float("nan"), dtype=torch.float32, device="cuda")
    # automatic split count, as the benchmark launches it
    ea.attn_fwd_ext(qg, kg, vg, o, lse, scale=scale_of(d), causal=True, window_left=wl,
                    alibi_slopes=sl, num_splits=0)
    torch.cuda.synchronize()
    assert ea.last_device_error() == 0
    rows = sample_rows(N + 17, B * H, N, 64)
    sl64 = [float(np.float32(x)) for x in slopes] if slopes else None
    o_ref, lse_ref = oracle.attention_ext(q, k, v, scale_of(d), True, wl, -1, sl64, rows=rows)
    e = compare(gather_rows(o.cpu(), rows), gather_rows(lse.cpu().unsqueeze(-1), rows).squeeze(-1),
                o_ref, lse_ref)
    assert_within(e, f"bench shape {(B, H, N, wl, alibi)}")
