"""The elementwise chain y = act(alpha * x + b), fused and unfused, against the
fp64 oracle on every element.

Bounds, from the arithmetic: the fused kernel computes in fp32 and rounds y
once to bf16, so |y - y_ref| <= 2^-8 |y_ref| plus fp32 noise (erf/exp to a few
fp32 ulps). The unfused path also rounds alpha * x and alpha * x + b to bf16
between its kernels; each rounding moves z = alpha * x + b by at most
2^-8 (|alpha x| + |z|) / 2 per step, and the activations' slopes are at most
1.13 (GELU, either form), 1.1 (SiLU), 1 (ReLU), so its bound adds
1.2 * 2^-8 (|alpha x| + |z|).
"""
import numpy as np
import pytest
import torch

import exact_attention_125_b200 as ea
import oracle

pytestmark = pytest.mark.gpu

U = 2.0 ** -8


def _inputs(rows, cols, seed):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn((rows, cols), generator=g).mul(2.5).to(torch.bfloat16)
    b = torch.randn((cols,), generator=g).to(torch.bfloat16)
    return x, b


@pytest.mark.parametrize("act", ["relu", "gelu", "silu", "gelu_tanh"])
@pytest.mark.parametrize("rows,cols", [(1, 8), (3, 24), (257, 136), (1000, 1024)])
def test_chain_fused_and_unfused(rows, cols, act):
    x, b = _inputs(rows, cols, rows * 7 + cols)
    alpha = -0.75
    y_ref = oracle.chain(x, b, alpha, act)
    xg, bg = x.cuda(), b.cuda()
    yf = ea.chain_fused(xg, bg, alpha=alpha, act=act)
    yu = ea.chain_unfused(xg, bg, alpha=alpha, act=act)
    torch.cuda.synchronize()
    ax = np.abs(alpha * x.double().numpy())
    z = alpha * x.double().numpy() + b.double().numpy()[None, :]
    ef = np.abs(yf.double().cpu().numpy() - y_ref)
    eu = np.abs(yu.double().cpu().numpy() - y_ref)
    assert (ef <= U * np.abs(y_ref) + 1e-6).all(), ef.max()
    assert (eu <= U * np.abs(y_ref) + 1.2 * U * (ax + np.abs(z)) + 1e-6).all(), eu.max()


def test_chain_large_tensor_sampled():
    # the benchmark's shape class: many rows, a wide hidden dimension; rows
    # sampled for the oracle
    x, b = _inputs(4096, 8192, 11)
    xg, bg = x.cuda(), b.cuda()
    yf = ea.chain_fused(xg, bg, alpha=0.5, act="gelu_tanh").cpu()
    rows = torch.tensor([0, 1, 777, 2048, 4095])
    y_ref = oracle.chain(x[rows], b, 0.5, "gelu_tanh")
    ef = np.abs(yf[rows].double().numpy() - y_ref)
    assert (ef <= U * np.abs(y_ref) + 1e-6).all()
