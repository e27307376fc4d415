"""The C-ABI library: it loads, exports every function include/attn.h
declares, and rejects bad arguments before any device work (no GPU needed)."""
import os
import re

import pytest

import exact_attention_125_b200 as ea
from exact_attention_125_b200 import _build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = [os.path.join(ROOT, "include", f) for f in sorted(os.listdir(os.path.join(ROOT, "include")))
           if f.endswith(".h")]


@pytest.fixture(scope="module")
def L():
    _build.build()
    return ea.lib()


def declared_functions():
    names = set()
    for h in HEADERS:
        text = re.sub(r"/\*.*?\*/", "", open(h).read(), flags=re.S)
        names |= set(re.findall(r"\b((?:attn|chain)_[a-z0-9_]+)\s*\(", text))
    return sorted(names)


def test_header_declares_the_boundary():
    names = declared_functions()
    for want in ("attn_fwd", "attn_fwd_naive", "attn_fwd_naive_workspace_bytes",
                 "attn_last_device_error", "attn_status_string", "attn_fwd_kv", "attn_fwd_ext",
                 "chain_fused", "chain_unfused"):
        assert want in names


def test_every_declared_symbol_is_exported(L):
    for name in declared_functions():
        assert hasattr(L, name), name


def test_status_strings(L):
    for code, name in ea.STATUS.items():
        assert ea.abi.attn_status_string(code).startswith(name)


A = 0x100000  # a 16-byte aligned fake device address; never dereferenced


def _fwd(**kw):
    args = dict(q=A, k=A, v=A, o=A, lse=A, B=1, H=1, N=128, d=64, scale=0.125, causal=0,
                stream=None)
    args.update(kw)
    return ea.abi.attn_fwd(args["q"], args["k"], args["v"], args["o"], args["lse"], args["B"],
                           args["H"], args["N"], args["d"], args["scale"], args["causal"],
                           args["stream"])


@pytest.mark.parametrize("kw,code", [
    (dict(q=None), -1), (dict(lse=None), -1),
    (dict(B=0), -2), (dict(N=0), -2), (dict(H=-3), -2), (dict(B=65536, H=65536), -2),
    (dict(d=96), -3), (dict(d=256), -3),
    (dict(q=A + 8), -4), (dict(o=A + 2), -4), (dict(lse=A + 2), -4),
    (dict(scale=float("nan")), -5), (dict(scale=float("inf")), -5),
    (dict(scale=float("-inf")), -5),
    (dict(causal=2), -6),
])
def test_fused_argument_errors(L, kw, code):
    assert _fwd(**kw) == code


def test_naive_argument_errors(L):
    n = ea.abi.attn_fwd_naive_workspace_bytes(1, 1, 128)
    assert n == 4 * 128 * 128
    assert ea.abi.attn_fwd_naive_workspace_bytes(8, 32, 8192) == 4 * 8 * 32 * 8192 * 8192
    assert ea.abi.attn_fwd_naive_workspace_bytes(0, 1, 1) == 0
    f = ea.abi.attn_fwd_naive
    assert f(A, A, A, A, A, 1, 1, 128, 64, 0.1, 0, None, n, None) == -1
    assert f(A, A, A, A, A, 1, 1, 128, 64, 0.1, 0, A + 4, n, None) == -4
    assert f(A, A, A, A, A, 1, 1, 128, 64, 0.1, 0, A, n - 1, None) == -7
    assert f(A, A, A, A, A, 1, 1, 40000, 64, 0.1, 0, A, 1 << 40, None) == -2


def test_wait_limit_is_settable(L):
    assert ea.wait_limit_ms() == 2000
    try:
        ea.set_wait_limit_ms(250)
        assert ea.wait_limit_ms() == 250
        for bad in (0, -5, 600001):
            with pytest.raises(ea.AttnError):
                ea.set_wait_limit_ms(bad)
        assert ea.wait_limit_ms() == 250
    finally:
        ea.set_wait_limit_ms(2000)


def test_selftest_argument_range(L):
    assert ea.abi.attn_selftest_wait_timeout(0, None) == -2
    assert ea.abi.attn_selftest_wait_timeout(6000, None) == -2


def test_product_path_has_no_fallback(monkeypatch):
    # with the library missing, the binding raises instead of computing
    monkeypatch.setattr(ea, "_lib", None)
    monkeypatch.setattr(ea, "_LIB_PATH", "/nonexistent/libattn_b200.so")
    with pytest.raises(RuntimeError):
        ea.lib()


def _kv(**kw):
    args = dict(q=A, k=A, v=A, o=A, lse=A, B=1, H=2, Nq=1, Nk=1000, d=128, scale=0.125,
                causal=0, splits=1, ws=None, ws_bytes=0, stream=None)
    args.update(kw)
    return ea.abi.attn_fwd_kv(args["q"], args["k"], args["v"], args["o"], args["lse"],
                              args["B"], args["H"], args["Nq"], args["Nk"], args["d"],
                              args["scale"], args["causal"], args["splits"], args["ws"],
                              args["ws_bytes"], args["stream"])


@pytest.mark.parametrize("kw,code", [
    (dict(k=None), -1), (dict(Nq=0), -2), (dict(Nk=0), -2), (dict(B=70000, H=70000), -2),
    (dict(Nq=5, Nk=4, causal=1), -2),           # causal needs Nq <= Nk
    (dict(d=80), -3), (dict(v=A + 4), -4), (dict(scale=float("nan")), -5), (dict(causal=3), -6),
    (dict(splits=-1), -2), (dict(splits=257), -2),
    (dict(splits=4), -1),                        # a split workspace is required
    (dict(splits=4, ws=A + 16, ws_bytes=1 << 30), -4),   # 256-byte alignment
    (dict(splits=4, ws=A, ws_bytes=100), -7),
])
def test_kv_argument_errors(L, kw, code):
    assert _kv(**kw) == code


def test_kv_workspace_bytes(L):
    f = ea.abi.attn_fwd_kv_workspace_bytes
    # 1000 keys = 8 tiles of 128; 4 splits of 2 tiles; [4][2][1][128] fp32 O + [4][2][1] lse
    assert f(1, 2, 1, 1000, 128, 4) == 4 * 2 * 128 * 4 + 4 * 2 * 4 + (256 - (4 * 2 * 128 * 4) % 256) % 256
    assert f(1, 2, 1, 1000, 128, 1) == 0
    # more splits than tiles clamp to the tile count; 3 requested on 8 tiles -> 3 tiles per
    # split -> 3 splits; 7 requested -> 2 tiles per split -> 4 splits (none empty)
    assert f(1, 1, 3, 1000, 64, 100) == f(1, 1, 3, 1000, 64, 8)
    assert f(1, 1, 3, 1000, 64, 7) == f(1, 1, 3, 1000, 64, 4)
    assert f(1, 1, 3, 1000, 64, 3) == 3 * 3 * 64 * 4 + 3 * 3 * 4 + (256 - (3 * 3 * 64 * 4) % 256) % 256
    assert f(0, 1, 3, 1000, 64, 3) == 0 and f(1, 1, 3, 1000, 96, 3) == 0


def _ext(**kw):
    args = dict(q=A, k=A, v=A, o=A, lse=A, B=1, H=2, Nq=4, Nk=1000, d=64, scale=0.125,
                causal=1, wl=127, wr=-1, slopes=None, splits=1, ws=None, ws_bytes=0, stream=None)
    args.update(kw)
    return ea.abi.attn_fwd_ext(*(args[n] for n in (
        "q", "k", "v", "o", "lse", "B", "H", "Nq", "Nk", "d", "scale", "causal", "wl", "wr",
        "slopes", "splits", "ws", "ws_bytes", "stream")))


@pytest.mark.parametrize("kw,code", [
    (dict(wl=-2), -12), (dict(wr=-5), -12), (dict(slopes=A + 2), -4), (dict(Nq=0), -2),
    (dict(splits=3), -1), (dict(splits=3, ws=A, ws_bytes=10), -7),
])
def test_ext_argument_errors(L, kw, code):
    assert _ext(**kw) == code


def test_ext_workspace_counts_only_the_window():
    f = ea.abi.attn_fwd_ext_workspace_bytes
    # 1 query row at position 999 with a 127-key left window reads keys 872..999:
    # tiles 6 and 7 only, so at most 2 splits
    assert f(1, 2, 1, 1000, 64, 127, 8) == f(1, 2, 1, 1000, 64, 127, 2)
    assert f(1, 2, 1, 1000, 64, 127, 2) == 2 * 2 * 64 * 4 + 2 * 2 * 4 + (256 - (2 * 2 * 64 * 4) % 256) % 256
    assert f(1, 2, 1, 1000, 64, -1, 8) == ea.abi.attn_fwd_kv_workspace_bytes(1, 2, 1, 1000, 64, 8)
    assert f(1, 2, 1, 1000, 64, -2, 8) == 0


def test_chain_argument_errors(L):
    f, u = ea.lib().chain_fused, ea.lib().chain_unfused
    import ctypes
    f.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_longlong, ctypes.c_int, ctypes.c_float,
                                          ctypes.c_int, ctypes.c_void_p]
    u.argtypes = [ctypes.c_void_p] * 4 + [ctypes.c_longlong, ctypes.c_int, ctypes.c_float,
                                          ctypes.c_int, ctypes.c_void_p]
    assert f(None, A, A, 4, 64, 1.0, 0, None) == -1
    assert f(A, A, A, 4, 60, 1.0, 0, None) == -2          # cols not a multiple of 8
    assert f(A, A, A, 0, 64, 1.0, 0, None) == -2
    assert f(A + 8, A, A, 4, 64, 1.0, 0, None) == -4
    assert f(A, A, A, 4, 64, float("nan"), 0, None) == -5
    assert f(A, A, A, 4, 64, 1.0, 4, None) == -6
    assert f(A, A, A, 4, 64, 1.0, -1, None) == -6
    assert u(A, A, A, None, 4, 64, 1.0, 1, None) == -1
    assert u(A, A, A, A + 4, 4, 64, 1.0, 1, None) == -4


def test_fp8_argument_errors(L):
    f = ea.abi.attn_fwd_fp8
    ok = dict(q=A, k=A, v=A, o=A, lse=A, B=1, H=1, N=128, d=128, scale=0.1, qd=0.01, kd=0.01,
              vd=0.01, causal=1, stream=None)

    def call(**kw):
        a = dict(ok, **kw)
        return f(a["q"], a["k"], a["v"], a["o"], a["lse"], a["B"], a["H"], a["N"], a["d"],
                 a["scale"], a["qd"], a["kd"], a["vd"], a["causal"], a["stream"])
    assert call(d=64) == -3                      # FP8 path: d = 128 only
    assert call(qd=0.0) == -5 and call(kd=float("inf")) == -5 and call(vd=-1.0) == -5
    assert call(v=None) == -1 and call(k=A + 1) == -4 and call(N=0) == -2 and call(causal=5) == -6
