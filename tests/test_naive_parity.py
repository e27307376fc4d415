"""attn_fwd_naive (three unfused kernels, S and P in HBM) against the oracle
and against the fused path."""
import pytest
import torch

import exact_attention_125_b200 as ea
from exact_attention_125_b200.inputs import WORKLOADS, make_qkv, make_workload
from parity_util import (check_naive_against_oracle, empty_outputs, sampled, scale_of,
                         to_gpu)

pytestmark = pytest.mark.gpu

SMALL = [
    (1, 1, 128, 64, False),
    (1, 1, 1, 64, True),
    (2, 1, 127, 64, True),
    (1, 2, 129, 128, False),
    (1, 1, 257, 128, True),
    (1, 2, 1000, 64, True),
]


def _run(q, k, v, scale, causal):
    qg, kg, vg = to_gpu(q, k, v)
    o, lse = empty_outputs(qg)
    ea.attn_fwd_naive(qg, kg, vg, o, lse, scale=scale, causal=causal)
    torch.cuda.synchronize()
    return o, lse


@pytest.mark.parametrize("B,H,N,d,causal", SMALL)
def test_small_shapes(B, H, N, d, causal):
    q, k, v = make_qkv(B, H, N, d, seed=N + d)
    o, lse = _run(q, k, v, scale_of(d), causal)
    check_naive_against_oracle(q, k, v, o, lse, scale_of(d), causal, what=f"naive {(B, H, N, d)}")


@pytest.mark.parametrize("scale", [0.0, -0.125])
@pytest.mark.parametrize("causal", [False, True])
def test_zero_and_negative_scale(scale, causal):
    q, k, v = make_qkv(1, 2, 300, 128, seed=41 + int(causal))
    o, lse = _run(q, k, v, scale, causal)
    check_naive_against_oracle(q, k, v, o, lse, scale, causal, what=f"naive scale {scale}")


def test_bert_base_all_rows():
    w = WORKLOADS["bert_base_1024"]
    q, k, v = make_workload(w)
    o, lse = _run(q, k, v, w.scale, w.causal)
    e = check_naive_against_oracle(q, k, v, o, lse, w.scale, w.causal, what="naive bert")
    print("naive", w.name, e)


def test_decoder_sampled():
    w = WORKLOADS["decoder_2048_causal"]
    q, k, v = make_workload(w)
    o, lse = _run(q, k, v, w.scale, w.causal)
    e = check_naive_against_oracle(q, k, v, o, lse, w.scale, w.causal, rows=sampled(w),
                                   what="naive dec")
    print("naive", w.name, e)


def test_naive_and_fused_agree():
    q, k, v = make_qkv(2, 4, 512, 128, seed=77)
    qg, kg, vg = to_gpu(q, k, v)
    o1, l1 = ea.attn_fwd(qg, kg, vg, causal=True)
    o2, l2 = ea.attn_fwd_naive(qg, kg, vg, causal=True)
    torch.cuda.synchronize()
    assert (o1.float() - o2.float()).abs().max().item() <= 2e-2
    assert (l1 - l2).abs().max().item() <= 1e-2


def test_workspace_too_small_is_rejected():
    q, k, v = to_gpu(*make_qkv(1, 1, 64, 64, seed=1))
    ws = torch.empty((ea.naive_workspace_bytes(1, 1, 64) - 16,), dtype=torch.uint8, device="cuda")
    with pytest.raises(ea.AttnError) as ei:
        ea.attn_fwd_naive(q, k, v, workspace=ws)
    assert ei.value.status == -7
