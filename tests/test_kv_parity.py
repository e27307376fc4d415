"""attn_fwd_kv (Nq query rows against Nk keys, key range split across CTAs and
merged by log-sum-exp) against the fp64 oracle, element by element.

Small and ragged shapes compare every row for explicit split counts and the
automatic one, covering both CTA layouts (Nq <= 128: one query tile whose two
softmax warpgroups take alternate KV tiles; Nq > 128: two query tiles sharing
every KV tile), splits in which some rows see no key at all, a single KV tile,
and Nq == Nk. The inference workloads compare a seeded row sample per head in
the launch configuration the benchmark times (automatic split count).
"""
import numpy as np
import pytest
import torch

import exact_attention_125_b200 as ea
import oracle
from exact_attention_125_b200.inputs import (KV_WORKLOADS, gather_rows, make_kv_workload,
                                             make_q_kv, sample_rows)
from parity_util import assert_within, compare, scale_of

pytestmark = pytest.mark.gpu

SMALL = [
    # B, H, Nq, Nk, d, causal, num_splits (0 = automatic)
    (1, 2, 1, 1000, 128, False, 1),
    (1, 2, 1, 1000, 128, False, 3),
    (1, 2, 1, 1000, 128, True, 0),
    (2, 3, 7, 1500, 64, True, 4),
    (1, 1, 128, 128, 128, True, 1),
    (1, 2, 100, 4097, 128, True, 5),
    (1, 2, 100, 1100, 128, True, 9),    # one tile per split; rows < 24 see none of the last
    (1, 2, 129, 700, 128, True, 2),
    (1, 2, 300, 2000, 64, False, 3),
    (1, 2, 300, 1000, 128, True, 8),    # rows < 68 / < 196 see nothing of splits 6 / 7
    (1, 1, 600, 600, 128, True, 1),
    (1, 1, 256, 5000, 128, True, 7),
    (2, 2, 33, 129, 64, False, 2),
    (1, 1, 1, 1, 128, False, 1),
    (1, 1, 5, 5, 64, True, 1),
    (1, 4, 64, 16384, 128, True, 0),
    (1, 3, 17, 3000, 64, False, 0),
]


def _run(q, k, v, scale, causal, splits):
    qg, kg, vg = (t.to("cuda") for t in (q, k, v))
    B, H, Nq, d = q.shape
    o = torch.full((B, H, Nq, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((B, H, Nq), float("nan"), dtype=torch.float32, device="cuda")
    ea.attn_fwd_kv(qg, kg, vg, o, lse, scale=scale, causal=causal, num_splits=splits)
    torch.cuda.synchronize()
    assert ea.last_device_error() == 0
    return o, lse


def _check(q, k, v, o, lse, scale, causal, rows, what):
    o_ref, lse_ref = oracle.attention_kv(q, k, v, scale, causal, rows=rows)
    o_rows = gather_rows(o.cpu(), rows)
    lse_rows = gather_rows(lse.cpu().unsqueeze(-1), rows).squeeze(-1)
    e = compare(o_rows, lse_rows, o_ref, lse_ref)
    assert_within(e, what)
    return e


@pytest.mark.parametrize("B,H,Nq,Nk,d,causal,splits", SMALL)
def test_small_shapes_all_rows(B, H, Nq, Nk, d, causal, splits):
    q, k, v = make_q_kv(B, H, Nq, Nk, d, seed=Nq * 31 + Nk + d + int(causal))
    o, lse = _run(q, k, v, scale_of(d), causal, splits)
    rows = oracle.all_rows(B * H, Nq)
    _check(q, k, v, o, lse, scale_of(d), causal, rows, f"{(B, H, Nq, Nk, d, causal, splits)}")


@pytest.mark.parametrize("scale", [0.0, -0.09])
@pytest.mark.parametrize("B,H,Nq,Nk,d,causal,splits", [
    (1, 2, 1, 1000, 128, False, 3),
    (1, 2, 100, 1100, 128, True, 9),
    (1, 2, 300, 2000, 64, False, 3),
])
def test_zero_and_negative_scale(B, H, Nq, Nk, d, causal, splits, scale):
    q, k, v = make_q_kv(B, H, Nq, Nk, d, seed=Nq * 31 + Nk + d + 5)
    o, lse = _run(q, k, v, scale, causal, splits)
    rows = oracle.all_rows(B * H, Nq)
    _check(q, k, v, o, lse, scale, causal, rows, f"{(B, H, Nq, Nk, d, causal, splits, scale)}")


def test_split_count_does_not_change_the_result_beyond_rounding():
    # every split count computes the same function; results differ only by
    # fp32 rounding order and the bf16 rounding of O
    q, k, v = make_q_kv(1, 2, 3, 5000, 128, seed=77)
    outs = [_run(q, k, v, 0.088, True, s) for s in (1, 2, 5, 40)]
    for o, lse in outs[1:]:
        assert (o.float() - outs[0][0].float()).abs().max().item() <= 2e-2
        assert (lse - outs[0][1]).abs().max().item() <= 1e-4 * 10


def test_square_problem_matches_attn_fwd():
    q, k, v = make_q_kv(1, 2, 700, 700, 128, seed=5)
    qg, kg, vg = (t.to("cuda") for t in (q, k, v))
    o1, l1 = ea.attn_fwd(qg, kg, vg, causal=True)
    o2, l2 = ea.attn_fwd_kv(qg, kg, vg, causal=True, num_splits=1)
    torch.cuda.synchronize()
    assert (o1.float() - o2.float()).abs().max().item() <= 1e-2
    assert (l1 - l2).abs().max().item() <= 1e-4


@pytest.mark.parametrize("name", list(KV_WORKLOADS))
def test_inference_workloads_sampled(name):
    w = KV_WORKLOADS[name]
    q, k, v = make_kv_workload(w)
    o, lse = _run(q, k, v, w.scale, w.causal, 0)
    rows = sample_rows(w.seed, w.B * w.H, w.Nq, w.rows_per_head)
    _check(q, k, v, o, lse, w.scale, w.causal, rows, name)
