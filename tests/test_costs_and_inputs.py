"""Host-side models and input generation (no GPU).

The byte model is pinned to the numbers printed on the anylearn.cc page
"Attention Is Memory-Bound, and Nobody Noticed for Five Years" (fixture
tests/golden/score_matrix_bytes.txt), each to the precision it is printed at.
"""
import os

import numpy as np
import pytest
import torch

from exact_attention_125_b200 import costs
from exact_attention_125_b200.inputs import (WORKLOADS, make_qkv, sample_rows,
                                             splitmix64)

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "score_matrix_bytes.txt")
UNITS = {"MB": 1e6, "GB": 1e9, "s": 1.0}


def _golden():
    for line in open(GOLDEN):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        kind, N, heads, batch, value, unit = line.split()
        yield kind, int(N), int(heads), int(batch), value, unit


def _decimals(s):
    return len(s.split(".")[1]) if "." in s else 0


@pytest.mark.parametrize("row", list(_golden()))
def test_printed_score_matrix_figures(row):
    kind, N, heads, batch, value, unit = row
    printed = float(value)
    if kind == "score_matrix":
        got = costs.score_matrix_bytes(N, heads, batch) / UNITS[unit]
        assert round(got, _decimals(value)) == printed
    elif kind == "four_crossings":
        # the page multiplies its rounded 34.4 GB by four and rounds again
        per = round(costs.score_matrix_bytes(N, heads, batch) / 1e9, 1)
        assert round(4 * per) == printed
        exact = costs.score_crossings_bytes(N, heads, batch) / UNITS[unit]
        assert abs(exact - printed) / printed < 0.005
    elif kind == "seconds_at_2TBps":
        t = costs.traffic_seconds(costs.score_crossings_bytes(N, heads, batch), 2e12)
        assert abs(t - printed) / printed < 0.05  # printed as "about 70 ms"
    else:
        raise AssertionError(kind)


def test_score_matrix_is_n_over_d_times_q():
    # the same page: the score matrix is larger than Q by a factor of n over d
    for N, d in ((8192, 64), (8192, 128), (2048, 64)):
        q_bytes = 2 * N * d
        assert costs.score_matrix_bytes(N) / q_bytes == N / d


def test_flop_convention():
    assert costs.attn_flops(1, 1, 128, 64, False) == 4 * 128 * 128 * 64
    assert costs.attn_flops(8, 32, 8192, 128, True) == pytest.approx(4.398e12, rel=1e-3)
    assert costs.attn_flops(1, 32, 65536, 128, True) == pytest.approx(3.518e13, rel=1e-3)


def test_fused_and_naive_bytes():
    assert costs.fused_bytes(8, 32, 8192, 128) == 8 * 8 * 32 * 8192 * 128 + 4 * 8 * 32 * 8192
    nb = costs.naive_kernel_bytes(8, 32, 8192, 128)
    assert sum(nb.values()) == costs.naive_bytes(8, 32, 8192, 128)
    # fused traffic is linear in N, naive quadratic
    assert costs.fused_bytes(1, 1, 2048, 64) == 2 * costs.fused_bytes(1, 1, 1024, 64)
    r = costs.naive_bytes(1, 1, 8192, 64) / costs.naive_bytes(1, 1, 4096, 64)
    assert 3.9 < r < 4.0


def test_tile_pairs():
    assert costs.tile_pairs(1, 1, 128, False) == 1
    assert costs.tile_pairs(1, 12, 1024, False) == 768
    assert costs.tile_pairs(8, 32, 2048, True) == 34816
    assert costs.tile_pairs(8, 32, 8192, True) == 532480
    assert costs.tile_pairs(1, 32, 65536, True) == 4202496


def test_splitmix64_published_values():
    # first outputs of SplitMix64 seeded with 0 (the reference sequence
    # published with the generator)
    z, s = splitmix64(0)
    assert z == 0xE220A8397B1DCDAF
    z, s = splitmix64(s)
    assert z == 0x6E789E6AA1B965F4


def test_make_qkv_is_seeded_and_bf16():
    a = make_qkv(1, 2, 8, 4, seed=3)
    b = make_qkv(1, 2, 8, 4, seed=3)
    c = make_qkv(1, 2, 8, 4, seed=4)
    for x, y in zip(a, b):
        assert x.dtype == torch.bfloat16 and x.is_contiguous() and torch.equal(x, y)
    assert not torch.equal(a[0], c[0])
    q, k, v = make_qkv(1, 1, 4096, 8, seed=5, dist="stress")
    assert 3.5 < q.float().std().item() < 4.5
    assert v.float().abs().max().item() <= 1.0
    g = make_qkv(1, 1, 64, 8, seed=5, dist="grid8")[1].float()
    assert torch.equal(g * 8, torch.round(g * 8)) and g.abs().max() <= 4


def test_sample_rows():
    r = sample_rows(1004, 3, 8192, 256)
    assert r.shape == (3 * 256, 2)
    for bh in range(3):
        rows = r[r[:, 0] == bh, 1]
        assert len(set(rows.tolist())) == 256
        assert rows[0] == 0 and rows[-1] == 8191 and (np.diff(rows) > 0).all()
    assert np.array_equal(r, sample_rows(1004, 3, 8192, 256))
    small = sample_rows(1, 2, 100, 256)
    assert small.shape == (200, 2)


def test_workload_table():
    w = WORKLOADS["long_8192_causal"]
    assert (w.B, w.H, w.N, w.d, w.causal) == (8, 32, 8192, 128, True)
    assert [x.seed for x in WORKLOADS.values()] == [1001, 1002, 1003, 1004, 1005]


@pytest.mark.parametrize("Nq,Nk", [(1, 1), (1, 9), (3, 10), (5, 5), (17, 300)])
def test_kv_visible_pairs_count_the_mask(Nq, Nk):
    i = np.arange(Nq)[:, None]
    j = np.arange(Nk)[None, :]
    assert costs.kv_visible_pairs(Nq, Nk, True) == int((j <= i + (Nk - Nq)).sum())
    assert costs.kv_visible_pairs(Nq, Nk, False) == Nq * Nk
    assert costs.kv_flops(2, 3, Nq, Nk, 64, True) == 4.0 * 2 * 3 * 64 * int((j <= i + (Nk - Nq)).sum())


def test_kv_bytes_decode_example():
    # one query row against 131072 keys, d = 128, 4 x 32 heads: K and V dominate
    b = costs.kv_bytes(4, 32, 1, 131072, 128)
    assert b == 128 * (2 * 128 * 2 + 2 * 131072 * 128 * 2 + 4)


def test_kv_inputs_shapes_and_determinism():
    from exact_attention_125_b200.inputs import make_q_kv
    q, k, v = make_q_kv(1, 2, 3, 7, 8, seed=5)
    assert q.shape == (1, 2, 3, 8) and k.shape == v.shape == (1, 2, 7, 8)
    q2, k2, v2 = make_q_kv(1, 2, 3, 7, 8, seed=5)
    assert torch.equal(q, q2) and torch.equal(k, k2) and torch.equal(v, v2)


@pytest.mark.parametrize("Nq,Nk,causal,wl,wr", [(5, 9, True, 2, -1), (7, 7, False, 1, 3),
                                                (3, 12, False, -1, 0), (6, 6, True, -1, -1)])
def test_ext_visible_pairs_count_the_mask(Nq, Nk, causal, wl, wr):
    pos = np.arange(Nq)[:, None] + (Nk - Nq)
    j = np.arange(Nk)[None, :]
    ok = np.ones((Nq, Nk), dtype=bool)
    if causal:
        ok &= j <= pos
    if wl >= 0:
        ok &= j >= pos - wl
    if wr >= 0:
        ok &= j <= pos + wr
    assert costs.ext_visible_pairs(Nq, Nk, causal, wl, wr) == int(ok.sum())
    if wl < 0 and wr < 0:
        assert costs.ext_visible_pairs(Nq, Nk, causal) == costs.kv_visible_pairs(Nq, Nk, causal)
