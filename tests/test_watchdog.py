"""The bounded-wait watchdog on the device: a wait on a barrier that nothing
ever arrives on gives up after its limit, records ATTN_ERR_TIMEOUT, and the
context stays usable (a normal launch afterwards succeeds)."""
import time

import pytest
import torch

import exact_attention_125_b200 as ea
from exact_attention_125_b200.inputs import make_qkv

pytestmark = pytest.mark.gpu


def test_wait_times_out_and_device_stays_usable():
    assert ea.last_device_error() == 0
    t0 = time.time()
    assert ea.selftest_wait_timeout(50) == 0
    torch.cuda.synchronize()
    assert time.time() - t0 < 5.0
    assert ea.last_device_error() == -10
    assert ea.last_device_error() == 0  # read clears it
    q, k, v = (t.cuda() for t in make_qkv(1, 1, 128, 64, seed=1))
    o, lse = ea.attn_fwd(q, k, v)
    torch.cuda.synchronize()
    assert torch.isfinite(o.float()).all()
    assert ea.last_device_error() == 0
