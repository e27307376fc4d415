"""Pins of the fp64 oracle against facts that do not come from the oracle.

Each test pins a part of the oracle to something independent: closed forms
derived by hand, invariants of the softmax definition, brute force through a
library softmax on tiny inputs, and exact-representability arguments. A
plausible slip in the oracle (a dropped scale, a mask off by one, a transposed
operand, a wrong log base, a missing max subtraction) fails at least one.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from exact_attention_125_b200.inputs import make_qkv

RNG = np.random.default_rng(12345)


def _rand(B, H, N, d, scale=1.0):
    return (RNG.standard_normal((B, H, N, d)) * scale for _ in range(3))


def _flat(o, B, H, N, d):
    return o.reshape(B, H, N, d)


def test_two_key_closed_form():
    # d = 1, N = 2, q = 1, keys chosen so the logits are s = (0, ln 3):
    # exp(s) = (1, 3), so p = (1/4, 3/4), o = p . v = 3/4 with v = (0, 1),
    # and lse = ln(1 + 3) = ln 4.
    scale = 0.37
    q = np.array([1.0, 1.0]).reshape(1, 1, 2, 1)
    k = np.array([0.0, math.log(3.0) / scale]).reshape(1, 1, 2, 1)
    v = np.array([0.0, 1.0]).reshape(1, 1, 2, 1)
    o, lse = oracle.attention(q, k, v, scale, causal=False)
    assert abs(o[0, 0] - 0.75) < 1e-15 and abs(o[1, 0] - 0.75) < 1e-15
    assert abs(lse[0] - math.log(4.0)) < 1e-15
    # causal: row 0 sees key 0 only (o = v0 = 0, lse = s00 = 0); row 1 sees both.
    o, lse = oracle.attention(q, k, v, scale, causal=True)
    assert o[0, 0] == 0.0 and lse[0] == 0.0
    assert abs(o[1, 0] - 0.75) < 1e-15 and abs(lse[1] - math.log(4.0)) < 1e-15


def test_large_logits_stay_finite():
    # logits (1000, 1000 + ln 3): a version without the max subtraction
    # overflows exp(); the exact answer is the same as the two-key case shifted.
    scale = 1.0
    q = np.array([1.0, 1.0]).reshape(1, 1, 2, 1)
    k = np.array([1000.0, 1000.0 + math.log(3.0)]).reshape(1, 1, 2, 1)
    v = np.array([0.0, 1.0]).reshape(1, 1, 2, 1)
    o, lse = oracle.attention(q, k, v, scale, causal=False)
    assert abs(o[0, 0] - 0.75) < 1e-13
    assert abs(lse[0] - (1000.0 + math.log(4.0))) < 1e-12


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N,d", [(1, 1), (2, 2), (5, 4), (16, 1), (13, 3)])
def test_brute_force_vs_torch_softmax(N, d, causal):
    # softmax(Q K^T * scale + mask) V through torch's own float64 softmax.
    B, H = 2, 3
    q, k, v = _rand(B, H, N, d)
    scale = 0.7
    o, lse = oracle.attention(q, k, v, scale, causal)
    tq, tk, tv = (torch.from_numpy(x) for x in (q, k, v))
    logits = torch.einsum("bhid,bhjd->bhij", tq, tk) * scale
    if causal:
        mask = torch.ones(N, N, dtype=torch.bool).triu(1)
        logits = logits.masked_fill(mask, float("-inf"))
    ref = torch.softmax(logits, dim=-1) @ tv
    ref_lse = torch.logsumexp(logits, dim=-1)
    assert np.abs(o - ref.numpy().reshape(-1, d)).max() <= 1e-12
    assert np.abs(lse - ref_lse.numpy().reshape(-1)).max() <= 1e-12


@pytest.mark.parametrize("causal", [False, True])
def test_scale_zero_is_mean_of_allowed_values(causal):
    # scale = 0 makes every allowed logit 0: each allowed key gets 1/|J(i)|,
    # so o_i = mean of v_0..v_i (causal) or of all v (non-causal) and
    # lse_i = ln |J(i)|. A mask that is off by one changes both.
    B, H, N, d = 1, 2, 9, 3
    q, k, v = _rand(B, H, N, d)
    o, lse = oracle.attention(q, k, v, 0.0, causal)
    o = o.reshape(B, H, N, d)
    lse = lse.reshape(B, H, N)
    for h in range(H):
        for i in range(N):
            n = i + 1 if causal else N
            assert np.abs(o[0, h, i] - v[0, h, :n].mean(axis=0)).max() < 1e-14
            assert abs(lse[0, h, i] - math.log(n)) < 1e-14


@pytest.mark.parametrize("causal", [False, True])
def test_constant_values_give_constant_output(causal):
    # each probability row sums to one, so V rows all equal to c give O = c;
    # with V = 1 this is the row-sum invariant itself.
    B, H, N, d = 2, 2, 17, 5
    q, k, _ = _rand(B, H, N, d, 2.0)
    c = RNG.standard_normal(d)
    v = np.broadcast_to(c, (B, H, N, d)).copy()
    o, _ = oracle.attention(q, k, v, 0.3, causal)
    assert np.abs(o - c).max() < 1e-13
    o1, _ = oracle.attention(q, k, np.ones_like(v), 0.3, causal)
    assert np.abs(o1 - 1.0).max() < 1e-14


def test_single_key():
    # N = 1: the only probability is 1, o = v0, lse = scale * q0 . k0.
    q, k, v = _rand(3, 2, 1, 6)
    o, lse = oracle.attention(q, k, v, 0.25, causal=False)
    assert np.abs(o - v.reshape(-1, 6)).max() == 0.0
    want = 0.25 * np.einsum("bhid,bhid->bhi", q, k).reshape(-1)
    assert np.abs(lse - want).max() < 1e-14


def test_causal_first_row_is_first_value():
    q, k, v = _rand(2, 2, 11, 4, 3.0)
    rows = np.array([[bh, 0] for bh in range(4)], dtype=np.int64)
    o, lse = oracle.attention(q, k, v, 0.5, True, rows=rows)
    assert np.abs(o - v[:, :, 0, :].reshape(4, 4)).max() == 0.0
    want = 0.5 * np.einsum("bhd,bhd->bh", q[:, :, 0], k[:, :, 0]).reshape(-1)
    assert np.abs(lse - want).max() < 1e-14


@pytest.mark.parametrize("causal", [False, True])
def test_per_row_logit_shift(causal):
    # K' = K + 1 u^T adds scale * (q_i . u) to every logit of row i: the
    # softmax is unchanged, lse shifts by exactly that amount.
    B, H, N, d = 1, 2, 12, 4
    q, k, v = _rand(B, H, N, d)
    u = RNG.standard_normal(d)
    scale = 0.6
    o, lse = oracle.attention(q, k, v, scale, causal)
    o2, lse2 = oracle.attention(q, k + u, v, scale, causal)
    shift = scale * (q @ u).reshape(-1)
    assert np.abs(o2 - o).max() < 1e-13
    assert np.abs(lse2 - lse - shift).max() < 1e-12


def test_key_permutation_invariance():
    # non-causal attention does not depend on the order of the (key, value)
    # pairs; a transposed or mis-indexed K or V breaks this.
    B, H, N, d = 1, 1, 10, 3
    q, k, v = _rand(B, H, N, d)
    perm = RNG.permutation(N)
    o, lse = oracle.attention(q, k, v, 0.8, False)
    o2, lse2 = oracle.attention(q, k[:, :, perm], v[:, :, perm], 0.8, False)
    assert np.abs(o - o2).max() < 1e-14 and np.abs(lse - lse2).max() < 1e-14


def test_asymmetric_scores_orientation():
    # s_ij = q_i . k_j, not q_j . k_i: with one query row much longer than the
    # keys, swapping the operands gives a different answer. Keys are 1-hot so
    # s_ij = q_i[j]; row 0 picks key 2 (logit 50), row 1 picks key 0.
    q = np.zeros((1, 1, 3, 3)); k = np.eye(3).reshape(1, 1, 3, 3)
    q[0, 0, 0] = [0.0, 0.0, 50.0]
    q[0, 0, 1] = [50.0, 0.0, 0.0]
    v = np.array([[1.0, 0, 0], [0, 1.0, 0], [0, 0, 1.0]]).reshape(1, 1, 3, 3)
    o, _ = oracle.attention(q, k, v, 1.0, False)
    assert o[0, 2] > 1 - 1e-15 and o[1, 0] > 1 - 1e-15
    assert o[0, 0] < 1e-20 and o[1, 2] < 1e-20
    # row 2 has q = 0: every logit is 0, uniform weights
    assert np.abs(o[2] - 1.0 / 3.0).max() < 1e-15


def test_probability_row_properties():
    N, d = 14, 5
    q = RNG.standard_normal((N, d))
    k = RNG.standard_normal((N, d))
    for causal in (False, True):
        for i in (0, 5, N - 1):
            p = oracle.probs_row(q, k, 0.4, causal, i)
            assert abs(p.sum() - 1.0) < 1e-15
            assert (p >= 0).all()
            if causal:
                assert (p[i + 1:] == 0).all() and (p[: i + 1] > 0).all()
            ref = torch.softmax(torch.from_numpy(q[i] @ k[: (i + 1 if causal else N)].T * 0.4), 0)
            assert np.abs(p[: len(ref)] - ref.numpy()).max() < 1e-15


def test_bf16_entry_widens_exactly():
    # The bf16 entry must give bit-identical results to the f64 entry fed
    # the same values (bf16 -> double is exact).
    q, k, v = make_qkv(2, 2, 37, 8, seed=7)
    o, lse = oracle.attention(q, k, v, 0.35, True)
    o2, lse2 = oracle.attention(q.double().numpy(), k.double().numpy(),
                                v.double().numpy(), 0.35, True)
    assert np.array_equal(o, o2) and np.array_equal(lse, lse2)


def test_sampled_rows_equal_full_rows_and_threads_agree():
    q, k, v = make_qkv(2, 3, 50, 8, seed=9)
    o_all, lse_all = oracle.attention(q, k, v, 0.3, True, nthreads=1)
    rows = np.array([[5, 49], [0, 0], [3, 17], [5, 3]], dtype=np.int64)
    o, lse = oracle.attention(q, k, v, 0.3, True, rows=rows, nthreads=4)
    flat = rows[:, 0] * 50 + rows[:, 1]
    assert np.array_equal(o, o_all[flat]) and np.array_equal(lse, lse_all[flat])
    o_mt, _ = oracle.attention(q, k, v, 0.3, True, nthreads=7)
    assert np.array_equal(o_mt, o_all)


def test_rejects_bad_rows():
    q, k, v = make_qkv(1, 1, 4, 2, seed=1)
    with pytest.raises(RuntimeError):
        oracle.attention(q, k, v, 1.0, False, rows=np.array([[0, 4]]))
    with pytest.raises(RuntimeError):
        oracle.attention(q, k, v, float("nan"), False)


# ----------------------------------------------------------------- Nq != Nk
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("Nq,Nk", [(1, 1), (1, 9), (3, 11), (7, 7), (5, 16)])
def test_kv_brute_force_vs_torch_softmax(Nq, Nk, causal):
    # queries are the last Nq of Nk positions: causally query i sees keys
    # j <= i + (Nk - Nq); brute force with torch's float64 softmax
    B, H, d = 2, 2, 4
    q = RNG.standard_normal((B, H, Nq, d))
    k = RNG.standard_normal((B, H, Nk, d))
    v = RNG.standard_normal((B, H, Nk, d))
    o, lse = oracle.attention_kv(q, k, v, 0.45, causal)
    tq, tk, tv = (torch.from_numpy(x) for x in (q, k, v))
    logits = torch.einsum("bhid,bhjd->bhij", tq, tk) * 0.45
    if causal:
        i = torch.arange(Nq)[:, None]
        j = torch.arange(Nk)[None, :]
        logits = logits.masked_fill(j > i + (Nk - Nq), float("-inf"))
    ref = torch.softmax(logits, dim=-1) @ tv
    assert np.abs(o - ref.numpy().reshape(-1, d)).max() <= 1e-12
    assert np.abs(lse - torch.logsumexp(logits, -1).numpy().reshape(-1)).max() <= 1e-12


def test_kv_queries_are_the_last_rows_of_full_attention():
    # the decode shape is the tail of the square problem: the last Nq rows of
    # causal attention over Nk positions equal Nq queries against Nk keys
    B, H, Nk, Nq, d = 1, 3, 40, 6, 5
    q_full = RNG.standard_normal((B, H, Nk, d))
    k = RNG.standard_normal((B, H, Nk, d))
    v = RNG.standard_normal((B, H, Nk, d))
    o_full, lse_full = oracle.attention(q_full, k, v, 0.3, True)
    o_tail, lse_tail = oracle.attention_kv(q_full[:, :, Nk - Nq:], k, v, 0.3, True)
    sel = np.concatenate([np.arange(bh * Nk + Nk - Nq, (bh + 1) * Nk) for bh in range(B * H)])
    assert np.array_equal(o_tail, o_full[sel]) and np.array_equal(lse_tail, lse_full[sel])
    # with Nq = Nk the two entry points are the same function
    o2, lse2 = oracle.attention_kv(q_full, k, v, 0.3, True)
    assert np.array_equal(o2, o_full) and np.array_equal(lse2, lse_full)


def test_kv_single_query_causal_sees_every_key():
    q = RNG.standard_normal((1, 2, 1, 4))
    k = RNG.standard_normal((1, 2, 13, 4))
    v = RNG.standard_normal((1, 2, 13, 4))
    o_c, l_c = oracle.attention_kv(q, k, v, 0.5, True)
    o_n, l_n = oracle.attention_kv(q, k, v, 0.5, False)
    assert np.array_equal(o_c, o_n) and np.array_equal(l_c, l_n)


# ------------------------------------------------ key windows, distance bias
def _ext_brute(q, k, v, scale, causal, wl, wr, slopes):
    B, H, Nq, d = q.shape
    Nk = k.shape[2]
    tq, tk, tv = (torch.from_numpy(x) for x in (q, k, v))
    logits = torch.einsum("bhid,bhjd->bhij", tq, tk) * scale
    pos = torch.arange(Nq)[:, None] + (Nk - Nq)
    j = torch.arange(Nk)[None, :]
    if slopes is not None:
        logits = logits - torch.tensor(slopes, dtype=torch.float64)[None, :, None, None] * \
            (pos - j).abs().to(torch.float64)
    allowed = torch.ones(Nq, Nk, dtype=torch.bool)
    if causal:
        allowed &= j <= pos
    if wl >= 0:
        allowed &= j >= pos - wl
    if wr >= 0:
        allowed &= j <= pos + wr
    logits = logits.masked_fill(~allowed, float("-inf"))
    return torch.softmax(logits, -1) @ tv, torch.logsumexp(logits, -1)


@pytest.mark.parametrize("causal,wl,wr,alibi", [
    (True, 3, -1, False), (False, 2, 1, False), (False, -1, 0, False), (False, 4, -1, True),
    (True, -1, -1, True), (True, 5, -1, True), (False, 0, 0, False), (False, 2, 3, True),
])
@pytest.mark.parametrize("Nq,Nk", [(1, 9), (6, 6), (4, 13)])
def test_ext_brute_force(Nq, Nk, causal, wl, wr, alibi):
    B, H, d = 2, 3, 4
    q = RNG.standard_normal((B, H, Nq, d))
    k = RNG.standard_normal((B, H, Nk, d))
    v = RNG.standard_normal((B, H, Nk, d))
    slopes = [0.5, 0.25, 0.125] if alibi else None
    o, lse = oracle.attention_ext(q, k, v, 0.4, causal, wl, wr, slopes)
    o_ref, lse_ref = _ext_brute(q, k, v, 0.4, causal, wl, wr, slopes)
    assert np.abs(o - o_ref.numpy().reshape(-1, d)).max() <= 1e-12
    assert np.abs(lse - lse_ref.numpy().reshape(-1)).max() <= 1e-12


def test_ext_without_options_is_attention_kv():
    q = RNG.standard_normal((1, 2, 5, 8))
    k = RNG.standard_normal((1, 2, 20, 8))
    v = RNG.standard_normal((1, 2, 20, 8))
    for causal in (False, True):
        o1, l1 = oracle.attention_kv(q, k, v, 0.3, causal)
        o2, l2 = oracle.attention_ext(q, k, v, 0.3, causal, -1, -1, None)
        o3, l3 = oracle.attention_ext(q, k, v, 0.3, causal, 100, 100, [0.0, 0.0])  # window covers all
        assert np.array_equal(o1, o2) and np.array_equal(l1, l2)
        assert np.array_equal(o1, o3) and np.array_equal(l1, l3)


def test_ext_diagonal_window_and_steep_bias_pick_the_own_position():
    # a window of width 0 leaves the query's own position: o = v[pos],
    # lse = scale q.k[pos]; a steep distance bias converges to the same o
    Nq, Nk, d = 4, 10, 6
    q = RNG.standard_normal((1, 1, Nq, d))
    k = RNG.standard_normal((1, 1, Nk, d))
    v = RNG.standard_normal((1, 1, Nk, d))
    pos = np.arange(Nq) + Nk - Nq
    o, lse = oracle.attention_ext(q, k, v, 0.5, False, 0, 0, None)
    assert np.array_equal(o, v[0, 0, pos])
    assert np.allclose(lse, 0.5 * np.einsum("id,id->i", q[0, 0], k[0, 0, pos]), rtol=0, atol=1e-15)
    # slope 60: the next key's weight is below exp(-60 + |logit differences|) ~ 1e-22
    o2, _ = oracle.attention_ext(q, k, v, 0.5, True, -1, -1, [60.0])
    assert np.abs(o2 - v[0, 0, pos]).max() <= 1e-15


def test_ext_bias_vanishes_at_the_own_position():
    # with a causal window of width 0 the only allowed key is the query's own
    # position, where the distance bias is slope * 0 = 0: nothing changes
    q = RNG.standard_normal((1, 1, 3, 4))
    k = RNG.standard_normal((1, 1, 7, 4))
    v = RNG.standard_normal((1, 1, 7, 4))
    o1, l1 = oracle.attention_ext(q, k, v, 0.5, True, 0, -1, None)
    o2, l2 = oracle.attention_ext(q, k, v, 0.5, True, 0, -1, [3.0])
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)  # |pos - pos| = 0


# --------------------------------------------------------- elementwise chain
def test_chain_closed_forms():
    # x = 2, b = -1, alpha = 0.5 -> z = 0 everywhere; x = 4, alpha = 0.5, b = 0 -> z = 2
    x = torch.tensor([[2.0, 4.0, -6.0, 1.0]], dtype=torch.bfloat16)
    b = torch.tensor([-1.0, 0.0, 1.0, 0.0], dtype=torch.bfloat16)
    z = np.array([0.0, 2.0, -2.0, 0.5])
    np.testing.assert_array_equal(oracle.chain(x, b, 0.5, "relu")[0], np.maximum(z, 0))
    g = oracle.chain(x, b, 0.5, "gelu")[0]
    # z Phi(z): Phi(0) = 1/2, Phi(2) = 0.9772498680518208, Phi(-2) = 1 - Phi(2)
    np.testing.assert_allclose(g, [0.0, 2 * 0.9772498680518208, -2 * (1 - 0.9772498680518208),
                                   0.5 * 0.6914624612740131], rtol=1e-15, atol=0)
    s = oracle.chain(x, b, 0.5, "silu")[0]
    np.testing.assert_allclose(s, z / (1 + np.exp(-z)), rtol=1e-15, atol=0)


@pytest.mark.parametrize("act", ["relu", "gelu", "silu", "gelu_tanh"])
def test_chain_matches_torch_float64(act):
    g = torch.Generator().manual_seed(3)
    x = torch.randn((5, 16), generator=g).mul(3).to(torch.bfloat16)
    b = torch.randn((16,), generator=g).to(torch.bfloat16)
    z = 1.75 * x.double() + b.double()
    ref = {"relu": torch.relu, "gelu": torch.nn.functional.gelu, "silu": torch.nn.functional.silu,
           "gelu_tanh": lambda t: torch.nn.functional.gelu(t, approximate="tanh")}[act](z)
    np.testing.assert_allclose(oracle.chain(x, b, 1.75, act), ref.numpy(), rtol=1e-14, atol=1e-15)


# -------------------------------------------------------------------- FP8
def test_e4m3_decoder_table_values():
    # sign, 4-bit exponent (bias 7), 3-bit mantissa; subnormals m * 2^-9; S.1111.111 = NaN
    assert oracle.e4m3_value(0x00) == 0.0
    assert oracle.e4m3_value(0x01) == 2.0 ** -9
    assert oracle.e4m3_value(0x07) == 7 * 2.0 ** -9
    assert oracle.e4m3_value(0x08) == 2.0 ** -6
    assert oracle.e4m3_value(0x38) == 1.0
    assert oracle.e4m3_value(0x3C) == 1.5
    assert oracle.e4m3_value(0x7E) == 448.0
    assert oracle.e4m3_value(0xFE) == -448.0
    assert oracle.e4m3_value(0x80) == 0.0 and np.signbit(oracle.e4m3_value(0x80))
    assert np.isnan(oracle.e4m3_value(0x7F)) and np.isnan(oracle.e4m3_value(0xFF))


def test_e4m3_decoder_matches_torch_for_all_codes():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = np.array([oracle.e4m3_value(c) for c in range(256)])
    nan = np.isnan(ref)
    assert (np.isnan(got) == nan).all()
    assert np.array_equal(got[~nan], ref[~nan])


@pytest.mark.parametrize("causal", [False, True])
def test_fp8_attention_is_attention_of_the_dequantized_tensors(causal):
    g = torch.Generator().manual_seed(21)
    q, k, v = (torch.randn((1, 2, 9, 8), generator=g).mul(40).to(torch.float8_e4m3fn) for _ in range(3))
    qd, kd, vd = 0.02, 0.03, 0.5
    o, lse = oracle.attention_fp8(q, k, v, 0.35, qd, kd, vd, causal)
    deq = [t.to(torch.float64).numpy() * s for t, s in ((q, qd), (k, kd), (v, vd))]
    o_ref, lse_ref = oracle.attention(*deq, 0.35, causal)
    assert np.abs(o - o_ref).max() <= 1e-13 * max(1.0, np.abs(o_ref).max())
    assert np.abs(lse - lse_ref).max() <= 1e-13 * max(1.0, np.abs(lse_ref).max())
