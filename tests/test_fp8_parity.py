"""attn_fwd_fp8 (E4M3 Q, K, V and P on the tensor cores) against the fp64 oracle
of the dequantized tensors, element by element.

Bound, from the arithmetic. The scores use the exact E4M3 inputs with fp32
accumulation, so S carries only fp32 rounding. The weights p = 2^(x - m)
(p <= 2^8 while the running max lags) are rounded to E4M3 before P V: to
nearest with relative error <= 2^-4 when p >= 2^-6, absolute error <= 2^-10
below (subnormals). With l the unrounded row sum (l >= 1 in the kernel's frame
and l >= sum_j e^(s_j - s_max) in any frame), an output element moves by at
most
    2^-4 * sum_j p_j |v_j| / l + 2^-10 * sum_j |v_j| / l
  <= 2^-4 * Oabs + 2^-10 * Vsum * e^(s_max - lse),
Oabs being attention of |V| and Vsum the sum of |v_j| over the allowed keys;
the bf16 output adds 2^-9 |O| (2^-8 |O| is used), the lse uses the unrounded
weights and keeps the common 1e-3 relative bound.
"""
import numpy as np
import pytest
import torch

import exact_attention_125_b200 as ea
import oracle
from exact_attention_125_b200.inputs import gather_rows, make_qkv_fp8, sample_rows

pytestmark = pytest.mark.gpu


def _abs_codes(t):
    return (t.view(torch.uint8) & 0x7F).view(torch.float8_e4m3fn)


def _check(q8, k8, v8, ds, scale, causal, rows, o, lse, what):
    qd, kd, vd = ds
    o_ref, lse_ref = oracle.attention_fp8(q8, k8, v8, scale, qd, kd, vd, causal, rows=rows)
    o_abs, _ = oracle.attention_fp8(q8, k8, _abs_codes(v8), scale, qd, kd, vd, causal, rows=rows)
    B, H, N, d = q8.shape
    qf = q8.to(torch.float64).reshape(B * H, N, d) * qd
    kf = k8.to(torch.float64).reshape(B * H, N, d) * kd
    vabs = v8.to(torch.float64).abs().reshape(B * H, N, d) * vd
    s_max = np.zeros(len(rows))
    vsum = np.zeros((len(rows), d))
    for r, (bh, i) in enumerate(rows):
        n = i + 1 if causal else N
        s_max[r] = float((scale * (kf[bh, :n] @ qf[bh, i])).max())
        vsum[r] = vabs[bh, :n].sum(0).numpy()
    got = gather_rows(o.cpu(), rows).double().numpy()
    got_lse = gather_rows(lse.cpu().unsqueeze(-1), rows).squeeze(-1).double().numpy()
    bound = (2.0 ** -4 * o_abs + 2.0 ** -10 * vsum * np.exp(s_max - lse_ref)[:, None]
             + 2.0 ** -8 * np.abs(o_ref) + 1e-4)
    err = np.abs(got - o_ref)
    assert np.isfinite(got).all(), what
    assert (err <= bound).all(), f"{what}: worst {err.max()} vs bound {bound[np.unravel_index(err.argmax(), err.shape)]}"
    lerr = np.abs(got_lse - lse_ref) / np.maximum(1.0, np.abs(lse_ref))
    assert lerr.max() <= 1e-3, f"{what}: lse {lerr.max()}"
    return err.max(), (err / np.maximum(np.abs(o_ref), 1e-3)).mean()


@pytest.mark.parametrize("B,H,N,causal", [(1, 2, 300, False), (1, 2, 300, True), (2, 3, 1000, True),
                                          (1, 1, 129, False), (1, 1, 1, True), (1, 2, 640, False),
                                          # more 256-row units than SMs: dealt in pairs
                                          (1, 80, 700, True)])
def test_fp8_small_all_rows(B, H, N, causal):
    (q8, k8, v8), ds = make_qkv_fp8(B, H, N, 128, seed=N + 5 * int(causal))
    o, lse = ea.attn_fwd_fp8(q8.cuda(), k8.cuda(), v8.cuda(), *ds, scale=128 ** -0.5, causal=causal)
    torch.cuda.synchronize()
    assert ea.last_device_error() == 0
    _check(q8, k8, v8, ds, 128 ** -0.5, causal, oracle.all_rows(B * H, N), o, lse, (B, H, N, causal))


@pytest.mark.parametrize("scale", [0.0, -(128 ** -0.5)])
def test_fp8_zero_and_negative_scale(scale):
    (q8, k8, v8), ds = make_qkv_fp8(1, 2, 300, 128, seed=71)
    o, lse = ea.attn_fwd_fp8(q8.cuda(), k8.cuda(), v8.cuda(), *ds, scale=scale, causal=True)
    torch.cuda.synchronize()
    assert ea.last_device_error() == 0
    _check(q8, k8, v8, ds, scale, True, oracle.all_rows(2, 300), o, lse, f"scale {scale}")


def test_fp8_long_sampled():
    B, H, N = 1, 4, 8192
    (q8, k8, v8), ds = make_qkv_fp8(B, H, N, 128, seed=99)
    o, lse = ea.attn_fwd_fp8(q8.cuda(), k8.cuda(), v8.cuda(), *ds, scale=128 ** -0.5, causal=True)
    torch.cuda.synchronize()
    assert ea.last_device_error() == 0
    rows = sample_rows(99, B * H, N, 48)
    _check(q8, k8, v8, ds, 128 ** -0.5, True, rows, o, lse, "long")
