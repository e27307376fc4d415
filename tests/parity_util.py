"""Comparison helpers for the GPU parity tests.

Tolerances are the ones the method is held to: on O, max-abs error <= 2e-2
and mean-abs error <= 2e-3 over every checked element; on the log-sum-exp,
|error| <= 1e-3 * max(1, |lse_ref|) (a relative bound that stays meaningful
when lse is near 0, e.g. the first causal row where lse = s_00).
"""
import numpy as np
import torch

import oracle
from exact_attention_125_b200.inputs import gather_rows, sample_rows

O_MAX_ABS = 2e-2
O_MEAN_ABS = 2e-3
LSE_REL = 1e-3
# unit roundoff of bf16 (8 significand bits, round to nearest even)
BF16_U = 2.0 ** -8


def compare(o_gpu_rows, lse_gpu_rows, o_ref, lse_ref):
    """Returns a dict of error figures; o_* are [R, d], lse_* are [R]."""
    o = o_gpu_rows.float().cpu().numpy().astype(np.float64)
    lse = lse_gpu_rows.float().cpu().numpy().astype(np.float64)
    err = np.abs(o - o_ref)
    lse_err = np.abs(lse - lse_ref) / np.maximum(1.0, np.abs(lse_ref))
    return {
        "o_max_abs": float(err.max()) if err.size else 0.0,
        "o_mean_abs": float(err.mean()) if err.size else 0.0,
        "lse_max_rel": float(lse_err.max()) if lse_err.size else 0.0,
        # plain relative error, for reporting (ill-conditioned where lse ~ 0)
        "lse_max_rel_plain": float((np.abs(lse - lse_ref) / np.abs(lse_ref)).max())
        if lse_err.size and (lse_ref != 0).all() else None,
        "finite": bool(np.isfinite(o).all() and np.isfinite(lse).all()),
    }


def assert_within(e, what="", lse=True):
    assert e["finite"], f"{what}: non-finite output {e}"
    assert e["o_max_abs"] <= O_MAX_ABS, f"{what}: O max-abs {e}"
    assert e["o_mean_abs"] <= O_MEAN_ABS, f"{what}: O mean-abs {e}"
    if lse:
        assert e["lse_max_rel"] <= LSE_REL, f"{what}: lse {e}"


def max_abs_logit(q, k, scale, causal, rows):
    """max over allowed keys j of |scale * q_i . k_j| for each (bh, i) row."""
    B, H, N, d = q.shape
    qf = q.reshape(B * H, N, d).double()
    kf = k.reshape(B * H, N, d).double()
    out = np.zeros(len(rows))
    for bh in np.unique(rows[:, 0]):
        sel = np.nonzero(rows[:, 0] == bh)[0]
        i = torch.as_tensor(rows[sel, 1])
        s = (qf[bh, i] @ kf[bh].T).abs() * abs(scale)
        if causal:
            s = s.masked_fill(torch.arange(N)[None, :] > i[:, None], 0.0)
        out[sel] = s.max(dim=1).values.numpy()
    return out


def check_naive_against_oracle(q, k, v, o, lse, scale, causal, rows=None, what=""):
    """The unfused path stores S in bf16 before the softmax, as the pages'
    16-bit score matrix does. Rounding each logit s_ij to bf16 moves it by at
    most delta_i = BF16_U * max_j |s_ij|, so lse_i, a smooth maximum of the
    logits, moves by at most delta_i (added to the lse tolerance), and each
    weight p_ij by a factor within e^(+-2 delta_i), so o_i moves by at most
    (e^(2 delta_i) - 1) * sum_j p_ij |v_j| (added to the per-element O
    max-abs bound; the O mean-abs bound is the common one)."""
    B, H, N, d = q.shape
    if rows is None:
        rows = oracle.all_rows(B * H, N)
    o_ref, lse_ref = oracle.attention(q, k, v, scale, causal, rows=rows)
    o_abs, _ = oracle.attention(q, k, v.abs(), scale, causal, rows=rows)
    o_rows = gather_rows(o.cpu(), rows)
    lse_rows = gather_rows(lse.cpu().unsqueeze(-1), rows).squeeze(-1)
    e = compare(o_rows, lse_rows, o_ref, lse_ref)
    delta = BF16_U * max_abs_logit(q, k, scale, causal, rows)
    o_err = np.abs(o_rows.double().numpy() - o_ref)
    o_bound = O_MAX_ABS + np.expm1(2.0 * delta)[:, None] * o_abs
    assert e["finite"], f"{what}: non-finite output {e}"
    assert (o_err <= o_bound).all(), f"{what}: naive O error {o_err.max()} vs bound {o_bound.flat[o_err.argmax()]}"
    assert e["o_mean_abs"] <= O_MEAN_ABS, f"{what}: O mean-abs {e}"
    bound = LSE_REL * np.maximum(1.0, np.abs(lse_ref)) + delta
    err = np.abs(lse_rows.double().numpy() - lse_ref)
    assert (err <= bound).all(), f"{what}: naive lse error {err.max()} vs bound {bound[err.argmax()]}"
    e["lse_max_abs"] = float(err.max())
    return e


def check_against_oracle(q, k, v, o, lse, scale, causal, rows=None, what=""):
    """q, k, v: CPU bf16 [B,H,N,d]; o, lse: GPU outputs. rows=None: all rows."""
    B, H, N, d = q.shape
    if rows is None:
        rows = oracle.all_rows(B * H, N)
    o_ref, lse_ref = oracle.attention(q, k, v, scale, causal, rows=rows)
    o_rows = gather_rows(o.cpu(), rows)
    lse_rows = gather_rows(lse.cpu().unsqueeze(-1), rows).squeeze(-1)
    e = compare(o_rows, lse_rows, o_ref, lse_ref)
    assert_within(e, what)
    return e


def sampled(w):
    return sample_rows(w.seed, w.B * w.H, w.N, 256)


def to_gpu(*ts):
    return tuple(t.to("cuda") for t in ts)


def scale_of(d):
    return 1.0 / float(np.sqrt(d))


def empty_outputs(q):
    B, H, N, d = q.shape
    o = torch.empty((B, H, N, d), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((B, H, N), dtype=torch.float32, device="cuda")
    return o, lse
