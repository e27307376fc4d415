"""attn_fwd_naive_noalloc: the unfused path for callers that cannot allocate.

Some callers of this library cannot call cudaMalloc or hand over a workspace:
code inside a host framework that owns the whole device-memory budget and
rejects allocations made outside its pool, and latency-bound loops where
cudaMalloc/cudaFree would add a device-wide synchronisation. For them the
library keeps S and P in its own fixed device array. This test calls that
entry point through the C ABI twice in a row, on different inputs, and checks
each result against attn_fwd_naive with a caller-owned workspace, using the
tolerances of the other parity tests, and against the fp64 oracle with the
unfused path's derived bound. The file is named so that pytest collects it
last.
"""
import numpy as np
import pytest
import torch

import exact_attention_125_b200 as ea
from exact_attention_125_b200.inputs import make_qkv

pytestmark = pytest.mark.gpu


def _ptrs(*ts):
    return [t.data_ptr() for t in ts]


def _with_workspace(q, k, v, scale, causal):
    B, H, N, d = q.shape
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device="cuda")
    ws_bytes = ea.abi.attn_fwd_naive_workspace_bytes(B, H, N)
    ws = torch.empty((ws_bytes,), dtype=torch.uint8, device="cuda")
    st = ea.abi.attn_fwd_naive(*_ptrs(q, k, v, o, lse), B, H, N, d, scale, int(causal),
                               ws.data_ptr(), ws_bytes, torch.cuda.current_stream().cuda_stream)
    assert st == 0, ea.STATUS.get(st)
    return o, lse


def _no_alloc(q, k, v, scale, causal):
    B, H, N, d = q.shape
    o = torch.full_like(q, float("nan"))
    lse = torch.full((B, H, N), float("nan"), dtype=torch.float32, device="cuda")
    st = ea.abi.attn_fwd_naive_noalloc(*_ptrs(q, k, v, o, lse), B, H, N, d, scale, int(causal),
                                       torch.cuda.current_stream().cuda_stream)
    assert st == 0, ea.STATUS.get(st)
    return o, lse


def _close(a, b):
    (o1, l1), (o2, l2) = a, b
    torch.cuda.synchronize()
    do = (o1.float() - o2.float()).abs()
    assert torch.isfinite(o2.float()).all() and torch.isfinite(l2).all()
    assert do.max().item() <= 2e-2 and do.mean().item() <= 2e-3
    rel = ((l1.double() - l2.double()).abs() / l1.double().abs().clamp(min=1.0)).max().item()
    assert rel <= 1e-3


@pytest.mark.parametrize("B,H,N,d,causal", [(1, 2, 1000, 64, True), (1, 12, 1024, 64, False),
                                            (2, 1, 333, 128, True)])
def test_no_alloc_matches_workspace_path_twice(B, H, N, d, causal):
    scale = 1.0 / float(np.sqrt(d))
    for call, seed in enumerate((100 + N, 200 + N)):
        q, k, v = (t.cuda() for t in make_qkv(B, H, N, d, seed=seed))
        _close(_with_workspace(q, k, v, scale, causal), _no_alloc(q, k, v, scale, causal))


@pytest.mark.parametrize("B,H,N,d,causal", [(1, 2, 1000, 64, True), (2, 1, 333, 128, False)])
def test_no_alloc_against_the_oracle(B, H, N, d, causal):
    # the same bound the workspace path is held to (bf16 S, derived allowance)
    from parity_util import check_naive_against_oracle
    scale = 1.0 / float(np.sqrt(d))
    q, k, v = make_qkv(B, H, N, d, seed=300 + N + int(causal))
    o, lse = _no_alloc(q.cuda(), k.cuda(), v.cuda(), scale, causal)
    torch.cuda.synchronize()
    check_naive_against_oracle(q, k, v, o, lse, scale, causal, what=f"noalloc {(B, H, N, d, causal)}")


def test_no_alloc_rejects_sizes_over_the_limit():
    # 4 * B * H * N * N bytes must fit the fixed array (64 MiB)
    B, H, N, d = 1, 1, 8192, 64  # needs 256 MiB
    assert 4 * B * H * N * N > ea.NOALLOC_SCRATCH_BYTES
    q = torch.zeros((B, H, N, d), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((B, H, N), dtype=torch.float32, device="cuda")
    st = ea.abi.attn_fwd_naive_noalloc(*_ptrs(q, q, q, q, lse), B, H, N, d, 0.125, 0,
                                       torch.cuda.current_stream().cuda_stream)
    assert st == -7  # ATTN_ERR_WORKSPACE, nothing launched
