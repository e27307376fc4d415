"""fp64 CPU oracle for exact scaled dot-product attention.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` use this module; the CUDA library never imports,
links or calls it, and it never imports the CUDA library.

The arithmetic lives in ``oracle.c`` (plain C, IEEE double, libm exp/log); this
file only builds that shared object with gcc and marshals numpy/torch arrays
into it.  It follows the three steps of standard attention named on the
grasp.study lesson "The Computational Steps of Standard Self-Attention"
(scores, row softmax, weighted sum of values) plus the log-sum-exp of each row.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

_CFLAGS = ["-O2", "-fPIC", "-shared", "-std=c11", "-Wall", "-Wextra",
           "-ffp-contract=off", "-pthread"]


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so next to it (gcc); returns the path."""
    if (not force and os.path.exists(_LIB)
            and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC)):
        return _LIB
    tmp = _LIB + f".tmp{os.getpid()}"
    subprocess.run(["gcc", *_CFLAGS, _SRC, "-o", tmp, "-lm"], check=True)
    os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        lib = ctypes.CDLL(build())
        i64p = ctypes.POINTER(ctypes.c_int64)
        f64p = ctypes.POINTER(ctypes.c_double)
        for name, elem in (("oracle_attn_bf16", ctypes.c_void_p),
                           ("oracle_attn_f64", ctypes.c_void_p)):
            fn = getattr(lib, name)
            fn.restype = ctypes.c_int
            fn.argtypes = [elem, elem, elem, ctypes.c_int, ctypes.c_int,
                           ctypes.c_int, ctypes.c_int, ctypes.c_double,
                           ctypes.c_int, i64p, ctypes.c_int64, f64p, f64p,
                           ctypes.c_int]
        for name in ("oracle_attn_kv_bf16", "oracle_attn_kv_f64"):
            fn = getattr(lib, name)
            fn.restype = ctypes.c_int
            fn.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int,
                           ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                           ctypes.c_double, ctypes.c_int, i64p, ctypes.c_int64, f64p, f64p,
                           ctypes.c_int]
        for name in ("oracle_attn_ext_bf16", "oracle_attn_ext_f64"):
            fn = getattr(lib, name)
            fn.restype = ctypes.c_int
            fn.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int,
                           ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                           ctypes.c_double, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                           ctypes.c_void_p, i64p, ctypes.c_int64, f64p, f64p, ctypes.c_int]
        lib.oracle_e4m3_to_double.restype = ctypes.c_double
        lib.oracle_e4m3_to_double.argtypes = [ctypes.c_uint8]
        lib.oracle_attn_e4m3.restype = ctypes.c_int
        lib.oracle_attn_e4m3.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                         ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                         ctypes.c_double, ctypes.c_double, ctypes.c_double,
                                         ctypes.c_double, ctypes.c_int, i64p, ctypes.c_int64,
                                         f64p, f64p, ctypes.c_int]
        lib.oracle_chain_bf16.restype = ctypes.c_int
        lib.oracle_chain_bf16.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64,
                                          ctypes.c_int, ctypes.c_double, ctypes.c_int, f64p]
        lib.oracle_probs_f64.restype = ctypes.c_int
        lib.oracle_probs_f64.argtypes = [f64p, f64p, ctypes.c_int, ctypes.c_int,
                                         ctypes.c_double, ctypes.c_int,
                                         ctypes.c_int, f64p]
        lib.oracle_default_threads.restype = ctypes.c_int
        lib.oracle_default_threads.argtypes = []
        _lib = lib
        return lib


def default_threads() -> int:
    """Number of host threads the oracle uses when not told otherwise."""
    return int(_load().oracle_default_threads())


def all_rows(BH: int, N: int) -> np.ndarray:
    """Every (bh, i) pair, shape [BH*N, 2] int64."""
    bh = np.repeat(np.arange(BH, dtype=np.int64), N)
    i = np.tile(np.arange(N, dtype=np.int64), BH)
    return np.stack([bh, i], axis=1)


def _as_bf16_bits(t) -> np.ndarray:
    """torch bf16 tensor (any device) -> contiguous numpy uint16 bit patterns."""
    import torch
    if not isinstance(t, torch.Tensor) or t.dtype != torch.bfloat16:
        raise TypeError("bf16 entry expects torch.bfloat16 tensors")
    return t.detach().to("cpu").contiguous().view(torch.int16).numpy().view(np.uint16)


def attention(q, k, v, scale: float, causal: bool, rows=None, nthreads: int = 0):
    """Exact attention rows in fp64.

    q, k, v: [B, H, N, d], either torch.bfloat16 tensors (the bf16 values are
    widened exactly) or float64 numpy arrays. rows: int64 array [R, 2] of
    (bh, i) pairs with bh = b*H + h, or None for every row.
    Returns (o [R, d] float64, lse [R] float64); lse is a natural logarithm.
    """
    lib = _load()
    if isinstance(q, np.ndarray):
        qa, ka, va = (np.ascontiguousarray(x, dtype=np.float64) for x in (q, k, v))
        fn = lib.oracle_attn_f64
    else:
        qa, ka, va = (_as_bf16_bits(x) for x in (q, k, v))
        fn = lib.oracle_attn_bf16
    if qa.ndim != 4 or ka.shape != qa.shape or va.shape != qa.shape:
        raise ValueError("q, k, v must share one [B, H, N, d] shape")
    B, H, N, d = (int(s) for s in qa.shape)
    if rows is None:
        rows = all_rows(B * H, N)
    rows = np.ascontiguousarray(rows, dtype=np.int64).reshape(-1, 2)
    R = rows.shape[0]
    o = np.zeros((R, d), dtype=np.float64)
    lse = np.zeros((R,), dtype=np.float64)
    st = fn(qa.ctypes.data, ka.ctypes.data, va.ctypes.data, B, H, N, d,
            float(scale), int(bool(causal)),
            rows.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), R,
            o.ctypes.data_as(ctypes.POINTER(ctypes.c_double)),
            lse.ctypes.data_as(ctypes.POINTER(ctypes.c_double)), int(nthreads))
    if st != 0:
        raise RuntimeError(f"oracle failed with status {st}")
    return o, lse


def attention_kv(q, k, v, scale: float, causal: bool, rows=None, nthreads: int = 0):
    """Nq queries against Nk keys: q [B, H, Nq, d], k and v [B, H, Nk, d]
    (torch.bfloat16 or float64 numpy). Causally, query i is position
    i + (Nk - Nq) of the sequence and sees keys j <= i + (Nk - Nq).
    rows: (bh, i) pairs with i < Nq, or None for all. Returns (o, lse)."""
    lib = _load()
    if isinstance(q, np.ndarray):
        qa, ka, va = (np.ascontiguousarray(x, dtype=np.float64) for x in (q, k, v))
        fn = lib.oracle_attn_kv_f64
    else:
        qa, ka, va = (_as_bf16_bits(x) for x in (q, k, v))
        fn = lib.oracle_attn_kv_bf16
    if qa.ndim != 4 or ka.shape != va.shape or ka.shape[:2] != qa.shape[:2] or ka.shape[3] != qa.shape[3]:
        raise ValueError("q [B, H, Nq, d] and k, v [B, H, Nk, d] expected")
    B, H, Nq, d = (int(x) for x in qa.shape)
    Nk = int(ka.shape[2])
    if rows is None:
        rows = all_rows(B * H, Nq)
    rows = np.ascontiguousarray(rows, dtype=np.int64).reshape(-1, 2)
    R = rows.shape[0]
    o = np.zeros((R, d), dtype=np.float64)
    lse = np.zeros((R,), dtype=np.float64)
    st = fn(qa.ctypes.data, ka.ctypes.data, va.ctypes.data, B, H, Nq, Nk, d, float(scale),
            int(bool(causal)), rows.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), R,
            o.ctypes.data_as(ctypes.POINTER(ctypes.c_double)),
            lse.ctypes.data_as(ctypes.POINTER(ctypes.c_double)), int(nthreads))
    if st != 0:
        raise RuntimeError(f"oracle failed with status {st}")
    return o, lse


def attention_ext(q, k, v, scale: float, causal: bool, window_left: int = -1,
                  window_right: int = -1, slopes=None, rows=None, nthreads: int = 0):
    """attention_kv with a key window and a linear distance bias. Query i is
    sequence position pos = i + Nk - Nq; key j is allowed iff j <= pos when
    causal, pos - window_left <= j when window_left >= 0 and j <= pos +
    window_right when window_right >= 0; with slopes (H values) the score of
    key j is lowered by slopes[h] * |pos - j|. Returns (o, lse)."""
    lib = _load()
    if isinstance(q, np.ndarray):
        qa, ka, va = (np.ascontiguousarray(x, dtype=np.float64) for x in (q, k, v))
        fn = lib.oracle_attn_ext_f64
    else:
        qa, ka, va = (_as_bf16_bits(x) for x in (q, k, v))
        fn = lib.oracle_attn_ext_bf16
    if qa.ndim != 4 or ka.shape != va.shape or ka.shape[:2] != qa.shape[:2] or ka.shape[3] != qa.shape[3]:
        raise ValueError("q [B, H, Nq, d] and k, v [B, H, Nk, d] expected")
    B, H, Nq, d = (int(x) for x in qa.shape)
    Nk = int(ka.shape[2])
    sl = None
    if slopes is not None:
        sl = np.ascontiguousarray(np.asarray(slopes, dtype=np.float64).reshape(-1))
        if sl.shape[0] != H:
            raise ValueError("one slope per head expected")
    if rows is None:
        rows = all_rows(B * H, Nq)
    rows = np.ascontiguousarray(rows, dtype=np.int64).reshape(-1, 2)
    R = rows.shape[0]
    o = np.zeros((R, d), dtype=np.float64)
    lse = np.zeros((R,), dtype=np.float64)
    st = fn(qa.ctypes.data, ka.ctypes.data, va.ctypes.data, B, H, Nq, Nk, d, float(scale),
            int(bool(causal)), int(window_left), int(window_right),
            sl.ctypes.data if sl is not None else None,
            rows.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), R,
            o.ctypes.data_as(ctypes.POINTER(ctypes.c_double)),
            lse.ctypes.data_as(ctypes.POINTER(ctypes.c_double)), int(nthreads))
    if st != 0:
        raise RuntimeError(f"oracle failed with status {st}")
    return o, lse


def e4m3_value(code: int) -> float:
    """The value of one OCP FP8 E4M3 code (0..255), decoded by the oracle."""
    return float(_load().oracle_e4m3_to_double(int(code)))


def _as_e4m3_codes(t) -> np.ndarray:
    import torch
    if not isinstance(t, torch.Tensor) or t.dtype != torch.float8_e4m3fn:
        raise TypeError("FP8 entry expects torch.float8_e4m3fn tensors")
    return t.detach().to("cpu").contiguous().view(torch.uint8).numpy()


def attention_fp8(q, k, v, scale: float, q_descale: float, k_descale: float, v_descale: float,
                  causal: bool, rows=None, nthreads: int = 0):
    """Attention of the dequantized tensors q_descale * Q, k_descale * K,
    v_descale * V, for E4M3 torch tensors [B, H, N, d]. Returns (o, lse)."""
    lib = _load()
    qa, ka, va = (_as_e4m3_codes(x) for x in (q, k, v))
    if qa.ndim != 4 or ka.shape != qa.shape or va.shape != qa.shape:
        raise ValueError("q, k, v must share one [B, H, N, d] shape")
    B, H, N, d = (int(x) for x in qa.shape)
    if rows is None:
        rows = all_rows(B * H, N)
    rows = np.ascontiguousarray(rows, dtype=np.int64).reshape(-1, 2)
    R = rows.shape[0]
    o = np.zeros((R, d), dtype=np.float64)
    lse = np.zeros((R,), dtype=np.float64)
    st = lib.oracle_attn_e4m3(qa.ctypes.data, ka.ctypes.data, va.ctypes.data, B, H, N, d,
                              float(scale), float(q_descale), float(k_descale), float(v_descale),
                              int(bool(causal)), rows.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)),
                              R, o.ctypes.data_as(ctypes.POINTER(ctypes.c_double)),
                              lse.ctypes.data_as(ctypes.POINTER(ctypes.c_double)), int(nthreads))
    if st != 0:
        raise RuntimeError(f"oracle failed with status {st}")
    return o, lse


def probs_row(q: np.ndarray, k: np.ndarray, scale: float, causal: bool, i: int):
    """Probability row p[0..N-1] of query i for one head (q, k: [N, d] float64)."""
    lib = _load()
    q = np.ascontiguousarray(q, dtype=np.float64)
    k = np.ascontiguousarray(k, dtype=np.float64)
    N, d = q.shape
    p = np.zeros((N,), dtype=np.float64)
    f64p = ctypes.POINTER(ctypes.c_double)
    st = lib.oracle_probs_f64(q.ctypes.data_as(f64p), k.ctypes.data_as(f64p), N, d,
                              float(scale), int(bool(causal)), int(i),
                              p.ctypes.data_as(f64p))
    if st != 0:
        raise RuntimeError(f"oracle_probs_f64 failed with status {st}")
    return p


CHAIN_ACTS = {"relu": 0, "gelu": 1, "silu": 2, "gelu_tanh": 3}


def chain(x, b, alpha: float, act: str):
    """y = act(alpha * x + b) in double for bf16 torch tensors x [rows, cols]
    and b [cols] (the elementwise chain); returns a float64 numpy array."""
    lib = _load()
    xa = _as_bf16_bits(x).reshape(-1)
    ba = _as_bf16_bits(b).reshape(-1)
    rows, cols = int(x.shape[0]), int(x.shape[1])
    if ba.shape[0] != cols:
        raise ValueError("one bias per column expected")
    y = np.zeros((rows, cols), dtype=np.float64)
    st = lib.oracle_chain_bf16(xa.ctypes.data, ba.ctypes.data, rows, cols, float(alpha),
                               CHAIN_ACTS[act], y.ctypes.data_as(ctypes.POINTER(ctypes.c_double)))
    if st != 0:
        raise RuntimeError(f"oracle_chain_bf16 failed with status {st}")
    return y
