"""The FMA-pipe exponential used for part of the softmax.

2^x = 2^j * p(f), x = j + f with j the nearest integer (Cody-Waite range
reduction) and p the degree-3 minimax polynomial for 2^f on [-1/2, 1/2]
(Remez exchange, exact_attention_125_b200/csrc/gen_exp2_poly.py). Pinned on the
CPU against the defining properties of a minimax fit and against numpy's
float64 exp2, and on the GPU against the same bound.
"""
import importlib.util
import os
import re

import numpy as np
import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
GEN = os.path.join(ROOT, "exact_attention_125_b200", "csrc", "gen_exp2_poly.py")
HEADER = os.path.join(ROOT, "exact_attention_125_b200", "csrc", "exp2_poly.cuh")


def _gen():
    spec = importlib.util.spec_from_file_location("gen_exp2_poly", GEN)
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    return m


def _header_coeffs():
    text = open(HEADER).read()
    c = [float(v) for v in re.findall(r"kExp2C\d = ([-0-9.e]+)f;", text)]
    bound = float(re.search(r"kExp2PolyMaxRelErr = ([-0-9.e]+)f;", text).group(1))
    return c, bound


def test_header_matches_a_fresh_fit():
    assert _gen().main(["--check"]) == 0


def test_minimax_equioscillation():
    # a minimax fit of degree 3 has an error that reaches +-E at 5 points with
    # alternating signs, and no larger error anywhere in the interval
    g = _gen()
    c, err = g.remez()
    x = np.linspace(-0.5, 0.5, 400001)
    e = g._error(c, x)
    assert abs(np.abs(e).max() - err) < 1e-12
    ext = [i for i in range(1, len(x) - 1) if abs(e[i]) >= abs(e[i - 1]) and abs(e[i]) >= abs(e[i + 1])]
    ext = [0] + ext + [len(x) - 1]
    peaks = [e[i] for i in ext if abs(e[i]) > 0.999 * err]
    signs = np.sign(peaks)
    assert len(peaks) >= 5 and all(signs[i] != signs[i + 1] for i in range(len(signs) - 1))
    # better than the Taylor cubic of 2^f = e^(f ln 2) it replaces
    taylor = [1.0, np.log(2), np.log(2) ** 2 / 2, np.log(2) ** 3 / 6]
    assert err < np.abs(g._error(taylor, x)).max() / 5


def _emulate_fp32(x):
    """The device algorithm step by step in float32 (numpy)."""
    c, _ = _header_coeffs()
    c0, c1, c2, c3 = (np.float32(v) for v in c)
    x = np.maximum(x.astype(np.float32), np.float32(-125.0))
    magic = np.float32(12582912.0)
    t = (x + magic).astype(np.float32)
    j = (t - magic).astype(np.float32)
    f = (x - j).astype(np.float32)
    p = (f * c3 + c2).astype(np.float32)
    p = (p * f + c1).astype(np.float32)
    p = (p * f + c0).astype(np.float32)
    bits = (p.view(np.uint32).astype(np.uint64) + (t.view(np.uint32).astype(np.uint64) << 23))
    return (bits & 0xFFFFFFFF).astype(np.uint32).view(np.float32)


def test_fp32_algorithm_within_bound():
    _, bound = _header_coeffs()
    x = np.concatenate([np.linspace(-125.0, 10.0, 2_000_001), np.arange(-125, 11, dtype=np.float64),
                        np.arange(-125, 10) + 0.5]).astype(np.float32)
    y = _emulate_fp32(x).astype(np.float64)
    rel = np.abs(y / np.exp2(x.astype(np.float64)) - 1.0)
    assert rel.max() <= bound + 4e-7
    low = _emulate_fp32(np.array([-126.0, -1000.0, -np.inf], dtype=np.float32))
    assert (low > 0).all() and (low <= 2.0 ** -124).all()


@pytest.mark.gpu
def test_device_exp2_poly_within_bound():
    import exact_attention_125_b200 as ea
    _, bound = _header_coeffs()
    xs = np.concatenate([np.linspace(-125.0, 10.0, 1_000_001), np.arange(-125, 11),
                         np.arange(-125, 10) + 0.5, [0.0, -0.0]]).astype(np.float32)
    x = torch.from_numpy(xs).cuda()
    y = torch.empty_like(x)
    assert ea.abi.attn_selftest_exp2(x.data_ptr(), y.data_ptr(), x.numel(),
                                     torch.cuda.current_stream().cuda_stream) == 0
    torch.cuda.synchronize()
    yd = y.cpu().numpy().astype(np.float64)
    rel = np.abs(yd / np.exp2(xs.astype(np.float64)) - 1.0)
    assert rel.max() <= bound + 4e-7, rel.max()
    low = torch.tensor([-126.0, -1000.0, float("-inf")], device="cuda")
    yl = torch.empty_like(low)
    assert ea.abi.attn_selftest_exp2(low.data_ptr(), yl.data_ptr(), 3,
                                     torch.cuda.current_stream().cuda_stream) == 0
    torch.cuda.synchronize()
    assert (yl > 0).all() and (yl <= 2.0 ** -124).all()
