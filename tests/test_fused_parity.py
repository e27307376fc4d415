"""attn_fwd (fused tcgen05 kernel) against the fp64 oracle, element by element.

Small and ragged shapes compare every row; the large workloads compare a
seeded sample of 256 query rows per (batch, head), rows 0 and N-1 included,
in the same launch configuration the benchmark times.
"""
import numpy as np
import pytest
import torch

import exact_attention_125_b200 as ea
from exact_attention_125_b200.inputs import WORKLOADS, make_qkv, make_workload
from parity_util import (check_against_oracle, empty_outputs, sampled, scale_of,
                         to_gpu)

pytestmark = pytest.mark.gpu

# With at most half as many 256-row work units as SMs, attn_fwd runs one
# 128-row query tile per CTA (its two softmax groups split the keys): these
# shapes check that layout.
SMALL = [
    # B, H, N, d, causal
    (1, 1, 128, 64, False),
    (1, 1, 128, 128, True),
    (1, 1, 1, 64, False),
    (1, 1, 1, 128, True),
    (1, 2, 2, 64, True),
    (2, 1, 127, 64, True),
    (1, 1, 129, 128, False),
    (1, 2, 255, 128, True),
    (1, 1, 257, 64, False),
    (1, 1, 1000, 128, True),
    (2, 3, 384, 128, False),
    (1, 2, 640, 64, True),
    (1, 1, 1000, 64, False),
    # several 256-row blocks with a ragged last one
    (1, 2, 1300, 128, True),
    (2, 1, 1536, 128, False),
    (1, 1, 2049, 128, True),
    (1, 1, 600, 128, False),
]


def _run(q, k, v, scale, causal):
    qg, kg, vg = to_gpu(q, k, v)
    o, lse = empty_outputs(qg)
    ea.attn_fwd(qg, kg, vg, o, lse, scale=scale, causal=causal)
    torch.cuda.synchronize()
    assert ea.last_device_error() == 0
    return o, lse


# Enough (batch, head) pairs that the 256-row work units outnumber the SMs,
# so the persistent kernel deals them to its CTAs in (heaviest, lightest)
# pairs across several units per CTA, carrying each next unit's first K tile
# in the previous unit's last ring unit; an odd number of blocks per head (the
# middle block forms a pair alone) and a ragged last block.
MANY_UNITS = [
    # B, H, N, d, causal
    (2, 40, 700, 128, True),
    (2, 40, 700, 64, False),
    (1, 80, 1100, 128, True),
]


# The same edge cases (one key, two keys, a ragged last tile, a query tile b
# past N) with enough heads that the persistent 256-row kernel runs them.
SQUARE_EDGES = [
    # B, H, N, d, causal
    (1, 160, 1, 64, False),
    (1, 160, 2, 128, True),
    (1, 80, 127, 64, True),
    (1, 80, 129, 128, False),
    (1, 80, 257, 64, True),
    (2, 40, 255, 128, False),
]


@pytest.mark.parametrize("B,H,N,d,causal", SQUARE_EDGES)
def test_square_kernel_edges_all_rows(B, H, N, d, causal):
    q, k, v = make_qkv(B, H, N, d, seed=7 * N + H + d + int(causal))
    o, lse = _run(q, k, v, scale_of(d), causal)
    check_against_oracle(q, k, v, o, lse, scale_of(d), causal, what=f"{(B, H, N, d, causal)}")


@pytest.mark.parametrize("B,H,N,d,causal", MANY_UNITS)
def test_many_units_odd_blocks_all_rows(B, H, N, d, causal):
    q, k, v = make_qkv(B, H, N, d, seed=3 * N + d + int(causal))
    o, lse = _run(q, k, v, scale_of(d), causal)
    check_against_oracle(q, k, v, o, lse, scale_of(d), causal, what=f"{(B, H, N, d, causal)}")


@pytest.mark.parametrize("B,H,N,d,causal", SMALL)
def test_small_shapes_all_rows(B, H, N, d, causal):
    q, k, v = make_qkv(B, H, N, d, seed=N * 7 + d + int(causal))
    o, lse = _run(q, k, v, scale_of(d), causal)
    check_against_oracle(q, k, v, o, lse, scale_of(d), causal, what=f"{(B, H, N, d, causal)}")


@pytest.mark.parametrize("name", ["single_head_128", "bert_base_1024", "decoder_2048_causal"])
def test_workloads_all_rows(name):
    w = WORKLOADS[name]
    q, k, v = make_workload(w)
    o, lse = _run(q, k, v, w.scale, w.causal)
    e = check_against_oracle(q, k, v, o, lse, w.scale, w.causal, what=name)
    print(name, e)


@pytest.mark.parametrize("name", ["long_8192_causal", "stress_65536_causal"])
def test_workloads_sampled_rows(name):
    w = WORKLOADS[name]
    q, k, v = make_workload(w)
    o, lse = _run(q, k, v, w.scale, w.causal)
    e = check_against_oracle(q, k, v, o, lse, w.scale, w.causal, rows=sampled(w), what=name)
    print(name, e)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d", [64, 128])
def test_constant_values(d, causal):
    # V rows all equal to c: every O row is c (probability rows sum to 1).
    B, H, N = 1, 2, 300
    q, k, _ = make_qkv(B, H, N, d, seed=5)
    c = torch.linspace(-2, 2, d).to(torch.bfloat16)
    v = c.expand(B, H, N, d).contiguous()
    o, _ = _run(q, k, v, scale_of(d), causal)
    err = (o.float().cpu() - c.float()).abs().max().item()
    assert err <= 2e-2


@pytest.mark.parametrize("d", [64, 128])
def test_single_key_and_causal_first_row(d):
    q, k, v = make_qkv(1, 3, 1, d, seed=11)
    o, lse = _run(q, k, v, scale_of(d), False)
    assert torch.equal(o.cpu(), v)  # exactly v0: p = 1, bf16 round trip exact
    want = (q.double() * k.double()).sum(-1) * scale_of(d)
    assert (lse.cpu().double() - want).abs().max().item() <= 1e-3 * max(1.0, want.abs().max().item())
    q, k, v = make_qkv(2, 2, 333, d, seed=12)
    o, _ = _run(q, k, v, scale_of(d), True)
    assert torch.equal(o[:, :, 0].cpu(), v[:, :, 0])


@pytest.mark.parametrize("causal", [False, True])
def test_per_row_logit_shift(causal):
    # K' = K + 1 u^T with entries on the 1/8 grid (exact in bf16): O is
    # unchanged and lse moves by scale * q_i . u (exact in the oracle).
    B, H, N, d = 1, 2, 260, 128
    q, k, v = make_qkv(B, H, N, d, seed=21, dist="grid8")
    u = make_qkv(1, 1, 1, d, seed=22, dist="grid8")[0].reshape(d)
    k2 = (k.float() + u.float()).to(torch.bfloat16)
    assert torch.equal(k2.float(), k.float() + u.float())
    scale = scale_of(d)
    o1, l1 = _run(q, k, v, scale, causal)
    o2, l2 = _run(q, k2, v, scale, causal)
    shift = (q.double() @ u.double()) * scale
    assert (o1.float() - o2.float()).abs().max().item() <= 2e-2
    dl = (l2.cpu().double() - l1.cpu().double() - shift).abs()
    assert dl.max().item() <= 1e-3 * max(1.0, l1.abs().max().item())


def test_outputs_do_not_depend_on_stale_memory():
    # outputs are fully overwritten: prefill with NaN, compare two runs
    q, k, v = make_qkv(1, 2, 200, 64, seed=3)
    qg, kg, vg = to_gpu(q, k, v)
    o = torch.full((1, 2, 200, 64), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((1, 2, 200), float("nan"), dtype=torch.float32, device="cuda")
    ea.attn_fwd(qg, kg, vg, o, lse, causal=True)
    o2, l2 = ea.attn_fwd(qg, kg, vg, causal=True)
    torch.cuda.synchronize()
    assert torch.equal(o, o2) and torch.equal(lse, l2)
    assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()


@pytest.mark.parametrize("H", [2, 80])  # the one-tile layout and the 256-row kernel
@pytest.mark.parametrize("scale", [0.0, -0.125, -1.0])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d", [64, 128])
def test_zero_and_negative_scale(d, causal, scale, H):
    # any finite scale is accepted; a negative one favours the smallest q.k
    q, k, v = make_qkv(1, H, 333, d, seed=31 + d + int(causal))
    o, lse = _run(q, k, v, scale, causal)
    check_against_oracle(q, k, v, o, lse, scale, causal, what=f"scale {scale}, d {d}")
    if scale == 0.0:
        # closed form: the mean of the allowed values, lse = ln |allowed keys|
        n = torch.arange(1, 334, dtype=torch.float64) if causal else torch.full((333,), 333.0,
                                                                                 dtype=torch.float64)
        vd = v.double()
        mean = (vd.cumsum(2) / n[:, None]) if causal else vd.mean(2, keepdim=True).expand_as(vd)
        assert (o.cpu().double() - mean).abs().max().item() <= 2e-2
        assert (lse.cpu().double() - n.log()).abs().max().item() <= 1e-3 * np.log(333.0)
