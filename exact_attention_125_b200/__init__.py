"""B200-native (sm_100a) exact attention forward.

Python binding of the C ABI in include/attn.h (libattn_b200.so, built in this
directory). This module only marshals arguments: every step of the attention
computation runs in the library's CUDA kernels. There is no CPU fallback; if
the library is missing, every call raises.

The torch-facing helpers take CUDA tensors (bf16 [B, H, N, d] for attention,
E4M3 for the FP8 path, bf16 [rows, cols] for the elementwise chain) and
allocate outputs and workspaces with torch when none are given (the library
never allocates):

  attn_fwd        fused forward, square problem (causal or not)
  attn_fwd_kv     Nq queries against Nk keys, key range split across CTAs
  attn_fwd_ext    attn_fwd_kv with key windows and a per-head distance bias
  attn_fwd_fp8    fused forward on E4M3 inputs with per-tensor scales
  attn_fwd_naive  the unfused three-kernel path (S and P through HBM)
  chain_fused / chain_unfused   act(alpha x + b) in one kernel or three
"""
from __future__ import annotations

import ctypes
import math
import os
import threading

__all__ = [
    "AttnError", "lib", "attn_fwd", "attn_fwd_kv", "kv_num_splits", "kv_workspace_bytes",
    "attn_fwd_ext", "ext_num_splits", "ext_workspace_bytes", "chain_fused", "chain_unfused",
    "attn_fwd_fp8",
    "CHAIN_ACTS",
    "attn_fwd_naive", "naive_workspace_bytes",
    "last_device_error", "status_string", "selftest_wait_timeout", "set_wait_limit_ms",
    "wait_limit_ms", "abi",
    "NOALLOC_SCRATCH_BYTES",
]

# Size of the library-owned scratch array behind attn_fwd_naive_noalloc
# (ATTN_NOALLOC_SCRATCH_BYTES in include/attn.h).
NOALLOC_SCRATCH_BYTES = 64 * 1024 * 1024

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libattn_b200.so")
_lock = threading.Lock()
_lib = None

ATTN_OK = 0
STATUS = {
    0: "ATTN_OK", -1: "ATTN_ERR_NULL", -2: "ATTN_ERR_SHAPE", -3: "ATTN_ERR_HEADDIM",
    -4: "ATTN_ERR_ALIGN", -5: "ATTN_ERR_SCALE", -6: "ATTN_ERR_CAUSAL",
    -7: "ATTN_ERR_WORKSPACE", -8: "ATTN_ERR_LAUNCH", -9: "ATTN_ERR_UNSUPPORTED_DEVICE",
    -10: "ATTN_ERR_TIMEOUT", -11: "ATTN_ERR_CUDA", -12: "ATTN_ERR_WINDOW",
}


class AttnError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)} ({status})")


def lib() -> ctypes.CDLL:
    """The loaded libattn_b200.so (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError(
                f"libattn_b200.so not found at {_LIB_PATH}; build it with "
                "`python -m exact_attention_125_b200._build` (no CPU fallback exists)")
        L = ctypes.CDLL(_LIB_PATH)
        vp, i, f, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
        L.attn_fwd.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, f, i, vp]
        L.attn_fwd.restype = i
        L.attn_fwd_fp8.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, f, f, f, f, i, vp]
        L.attn_fwd_fp8.restype = i
        L.attn_fwd_kv.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, f, i, i, vp, sz, vp]
        L.attn_fwd_kv.restype = i
        L.attn_fwd_kv_num_splits.argtypes = [i, i, i, i, i]
        L.attn_fwd_kv_num_splits.restype = i
        L.attn_fwd_kv_workspace_bytes.argtypes = [i, i, i, i, i, i]
        L.attn_fwd_kv_workspace_bytes.restype = sz
        L.attn_fwd_ext.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, f, i, i, i, vp, i, vp, sz,
                                   vp]
        L.attn_fwd_ext.restype = i
        L.attn_fwd_ext_num_splits.argtypes = [i, i, i, i, i, i]
        L.attn_fwd_ext_num_splits.restype = i
        L.attn_fwd_ext_workspace_bytes.argtypes = [i, i, i, i, i, i, i]
        L.attn_fwd_ext_workspace_bytes.restype = sz
        ll = ctypes.c_longlong
        L.chain_fused.argtypes = [vp, vp, vp, ll, i, f, i, vp]
        L.chain_fused.restype = i
        L.chain_unfused.argtypes = [vp, vp, vp, vp, ll, i, f, i, vp]
        L.chain_unfused.restype = i
        L.attn_fwd_naive_workspace_bytes.argtypes = [i, i, i]
        L.attn_fwd_naive_workspace_bytes.restype = sz
        L.attn_fwd_naive.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, f, i, vp, sz, vp]
        L.attn_fwd_naive.restype = i
        L.attn_fwd_naive_noalloc.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, f, i, vp]
        L.attn_fwd_naive_noalloc.restype = i
        L.attn_last_device_error.argtypes = [vp]
        L.attn_last_device_error.restype = i
        L.attn_status_string.argtypes = [i]
        L.attn_status_string.restype = ctypes.c_char_p
        L.attn_selftest_wait_timeout.argtypes = [i, vp]
        L.attn_selftest_wait_timeout.restype = i
        L.attn_selftest_exp2.argtypes = [vp, vp, i, vp]
        L.attn_selftest_exp2.restype = i
        L.attn_set_wait_limit_ms.argtypes = [i]
        L.attn_set_wait_limit_ms.restype = i
        L.attn_wait_limit_ms.argtypes = []
        L.attn_wait_limit_ms.restype = i
        _lib = L
        return L


class abi:
    """The C entry points with raw pointers and sizes, same names as attn.h."""

    @staticmethod
    def attn_fwd(q, k, v, o, lse, B, H, N, d, scale, causal, stream) -> int:
        return lib().attn_fwd(q, k, v, o, lse, B, H, N, d, scale, causal, stream)

    @staticmethod
    def attn_fwd_fp8(q, k, v, o, lse, B, H, N, d, scale, q_descale, k_descale, v_descale, causal,
                     stream) -> int:
        return lib().attn_fwd_fp8(q, k, v, o, lse, B, H, N, d, scale, q_descale, k_descale,
                                  v_descale, causal, stream)

    @staticmethod
    def attn_fwd_kv(q, k, v, o, lse, B, H, Nq, Nk, d, scale, causal, num_splits, ws, ws_bytes,
                    stream) -> int:
        return lib().attn_fwd_kv(q, k, v, o, lse, B, H, Nq, Nk, d, scale, causal, num_splits, ws,
                                 ws_bytes, stream)

    @staticmethod
    def attn_fwd_kv_num_splits(B, H, Nq, Nk, d) -> int:
        return lib().attn_fwd_kv_num_splits(B, H, Nq, Nk, d)

    @staticmethod
    def attn_fwd_kv_workspace_bytes(B, H, Nq, Nk, d, num_splits) -> int:
        return int(lib().attn_fwd_kv_workspace_bytes(B, H, Nq, Nk, d, num_splits))

    @staticmethod
    def attn_fwd_ext(q, k, v, o, lse, B, H, Nq, Nk, d, scale, causal, window_left, window_right,
                     alibi_slopes, num_splits, ws, ws_bytes, stream) -> int:
        return lib().attn_fwd_ext(q, k, v, o, lse, B, H, Nq, Nk, d, scale, causal, window_left,
                                  window_right, alibi_slopes, num_splits, ws, ws_bytes, stream)

    @staticmethod
    def attn_fwd_ext_num_splits(B, H, Nq, Nk, d, window_left) -> int:
        return lib().attn_fwd_ext_num_splits(B, H, Nq, Nk, d, window_left)

    @staticmethod
    def attn_fwd_ext_workspace_bytes(B, H, Nq, Nk, d, window_left, num_splits) -> int:
        return int(lib().attn_fwd_ext_workspace_bytes(B, H, Nq, Nk, d, window_left, num_splits))

    @staticmethod
    def chain_fused(x, b, y, rows, cols, alpha, act, stream) -> int:
        return lib().chain_fused(x, b, y, rows, cols, alpha, act, stream)

    @staticmethod
    def chain_unfused(x, b, y, tmp, rows, cols, alpha, act, stream) -> int:
        return lib().chain_unfused(x, b, y, tmp, rows, cols, alpha, act, stream)

    @staticmethod
    def attn_fwd_naive(q, k, v, o, lse, B, H, N, d, scale, causal, ws, ws_bytes, stream) -> int:
        return lib().attn_fwd_naive(q, k, v, o, lse, B, H, N, d, scale, causal, ws, ws_bytes,
                                    stream)

    @staticmethod
    def attn_fwd_naive_workspace_bytes(B, H, N) -> int:
        return int(lib().attn_fwd_naive_workspace_bytes(B, H, N))

    @staticmethod
    def attn_fwd_naive_noalloc(q, k, v, o, lse, B, H, N, d, scale, causal, stream) -> int:
        return lib().attn_fwd_naive_noalloc(q, k, v, o, lse, B, H, N, d, scale, causal, stream)

    @staticmethod
    def attn_last_device_error(stream) -> int:
        return lib().attn_last_device_error(stream)

    @staticmethod
    def attn_status_string(status) -> str:
        return lib().attn_status_string(status).decode()

    @staticmethod
    def attn_selftest_wait_timeout(limit_ms, stream) -> int:
        return lib().attn_selftest_wait_timeout(limit_ms, stream)

    @staticmethod
    def attn_selftest_exp2(x, y, n, stream) -> int:
        return lib().attn_selftest_exp2(x, y, n, stream)

    @staticmethod
    def attn_set_wait_limit_ms(ms) -> int:
        return lib().attn_set_wait_limit_ms(ms)

    @staticmethod
    def attn_wait_limit_ms() -> int:
        return lib().attn_wait_limit_ms()


def status_string(status: int) -> str:
    return abi.attn_status_string(status)


def _stream_handle(stream):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _check_qkv(q, k, v):
    import torch
    for name, t in (("q", q), ("k", k), ("v", v)):
        if not isinstance(t, torch.Tensor) or not t.is_cuda:
            raise TypeError(f"{name} must be a CUDA tensor")
        if t.dtype != torch.bfloat16 or t.dim() != 4 or not t.is_contiguous():
            raise TypeError(f"{name} must be a contiguous bf16 [B, H, N, d] tensor")
    if not (q.shape == k.shape == v.shape):
        raise ValueError("q, k, v must have the same shape")
    return tuple(int(s) for s in q.shape)


def _outputs(q, o, lse):
    import torch
    B, H, N, d = q.shape
    if o is None:
        o = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    return o, lse


def attn_fwd(q, k, v, o=None, lse=None, scale=None, causal=False, stream=None):
    """Fused forward. Returns (o, lse); o is bf16 [B,H,N,d], lse fp32 [B,H,N]."""
    B, H, N, d = _check_qkv(q, k, v)
    o, lse = _outputs(q, o, lse)
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    st = abi.attn_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                      B, H, N, d, scale, int(bool(causal)), _stream_handle(stream))
    if st != ATTN_OK:
        raise AttnError(st, "attn_fwd")
    return o, lse


def attn_fwd_fp8(q, k, v, q_descale, k_descale, v_descale, o=None, lse=None, scale=None,
                 causal=False, stream=None):
    """FP8 forward: q, k, v are CUDA torch.float8_e4m3fn tensors [B, H, N, 128]
    holding Q / q_descale etc. Returns (o bf16 [B, H, N, 128], lse fp32)."""
    import torch
    for name, t in (("q", q), ("k", k), ("v", v)):
        if not isinstance(t, torch.Tensor) or not t.is_cuda:
            raise TypeError(f"{name} must be a CUDA tensor")
        if t.dtype != torch.float8_e4m3fn or t.dim() != 4 or not t.is_contiguous():
            raise TypeError(f"{name} must be a contiguous float8_e4m3fn [B, H, N, d] tensor")
    if not (q.shape == k.shape == v.shape):
        raise ValueError("q, k, v must have the same shape")
    B, H, N, d = (int(x) for x in q.shape)
    if o is None:
        o = torch.empty((B, H, N, d), dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    st = abi.attn_fwd_fp8(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                          B, H, N, d, scale, float(q_descale), float(k_descale), float(v_descale),
                          int(bool(causal)), _stream_handle(stream))
    if st != ATTN_OK:
        raise AttnError(st, "attn_fwd_fp8")
    return o, lse


def kv_num_splits(B: int, H: int, Nq: int, Nk: int, d: int) -> int:
    """Split count attn_fwd_kv picks for num_splits=0 on the current device."""
    st = abi.attn_fwd_kv_num_splits(B, H, Nq, Nk, d)
    if st < 1:
        raise AttnError(st, "attn_fwd_kv_num_splits")
    return st


def kv_workspace_bytes(B: int, H: int, Nq: int, Nk: int, d: int, num_splits: int = 0) -> int:
    return abi.attn_fwd_kv_workspace_bytes(B, H, Nq, Nk, d, num_splits)


def attn_fwd_kv(q, k, v, o=None, lse=None, scale=None, causal=False, num_splits=0,
                workspace=None, stream=None):
    """Nq query rows against Nk keys: q [B,H,Nq,d], k and v [B,H,Nk,d] (CUDA bf16,
    contiguous). Causal alignment is bottom-right (query i sees keys j <= i + Nk - Nq).
    num_splits=0 lets the library choose. Returns (o [B,H,Nq,d] bf16, lse [B,H,Nq] fp32)."""
    import torch
    for name, t in (("q", q), ("k", k), ("v", v)):
        if not isinstance(t, torch.Tensor) or not t.is_cuda:
            raise TypeError(f"{name} must be a CUDA tensor")
        if t.dtype != torch.bfloat16 or t.dim() != 4 or not t.is_contiguous():
            raise TypeError(f"{name} must be a contiguous bf16 [B, H, N, d] tensor")
    if k.shape != v.shape or k.shape[:2] != q.shape[:2] or k.shape[3] != q.shape[3]:
        raise ValueError("q [B, H, Nq, d] and k, v [B, H, Nk, d] expected")
    B, H, Nq, d = (int(x) for x in q.shape)
    Nk = int(k.shape[2])
    o, lse = _outputs(q, o, lse)
    need = kv_workspace_bytes(B, H, Nq, Nk, d, num_splits)
    if workspace is None and need > 0:
        workspace = torch.empty((need,), dtype=torch.uint8, device=q.device)
    ws_ptr = workspace.data_ptr() if workspace is not None else None
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    st = abi.attn_fwd_kv(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                         B, H, Nq, Nk, d, scale, int(bool(causal)), int(num_splits), ws_ptr,
                         ws_bytes, _stream_handle(stream))
    if st != ATTN_OK:
        raise AttnError(st, "attn_fwd_kv")
    return o, lse


def ext_num_splits(B: int, H: int, Nq: int, Nk: int, d: int, window_left: int = -1) -> int:
    st = abi.attn_fwd_ext_num_splits(B, H, Nq, Nk, d, window_left)
    if st < 1:
        raise AttnError(st, "attn_fwd_ext_num_splits")
    return st


def ext_workspace_bytes(B: int, H: int, Nq: int, Nk: int, d: int, window_left: int = -1,
                        num_splits: int = 0) -> int:
    return abi.attn_fwd_ext_workspace_bytes(B, H, Nq, Nk, d, window_left, num_splits)


def attn_fwd_ext(q, k, v, o=None, lse=None, scale=None, causal=False, window_left=-1,
                 window_right=-1, alibi_slopes=None, num_splits=0, workspace=None, stream=None):
    """attn_fwd_kv with a key window [pos - window_left, pos + window_right]
    around each query's position (-1 = unbounded) and an optional per-head
    linear distance bias (alibi_slopes: CUDA fp32 tensor of H slopes; the
    logit of key j drops by slope * |pos - j|). Returns (o, lse)."""
    import torch
    for name, t in (("q", q), ("k", k), ("v", v)):
        if not isinstance(t, torch.Tensor) or not t.is_cuda:
            raise TypeError(f"{name} must be a CUDA tensor")
        if t.dtype != torch.bfloat16 or t.dim() != 4 or not t.is_contiguous():
            raise TypeError(f"{name} must be a contiguous bf16 [B, H, N, d] tensor")
    if k.shape != v.shape or k.shape[:2] != q.shape[:2] or k.shape[3] != q.shape[3]:
        raise ValueError("q [B, H, Nq, d] and k, v [B, H, Nk, d] expected")
    B, H, Nq, d = (int(x) for x in q.shape)
    Nk = int(k.shape[2])
    sl_ptr = None
    if alibi_slopes is not None:
        if (not isinstance(alibi_slopes, torch.Tensor) or not alibi_slopes.is_cuda or
                alibi_slopes.dtype != torch.float32 or alibi_slopes.numel() != H or
                not alibi_slopes.is_contiguous()):
            raise TypeError("alibi_slopes must be a contiguous CUDA float32 tensor of H values")
        sl_ptr = alibi_slopes.data_ptr()
    o, lse = _outputs(q, o, lse)
    need = ext_workspace_bytes(B, H, Nq, Nk, d, window_left, num_splits)
    if workspace is None and need > 0:
        workspace = torch.empty((need,), dtype=torch.uint8, device=q.device)
    ws_ptr = workspace.data_ptr() if workspace is not None else None
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    st = abi.attn_fwd_ext(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                          B, H, Nq, Nk, d, scale, int(bool(causal)), int(window_left),
                          int(window_right), sl_ptr, int(num_splits), ws_ptr, ws_bytes,
                          _stream_handle(stream))
    if st != ATTN_OK:
        raise AttnError(st, "attn_fwd_ext")
    return o, lse


# CHAIN_ACT_* of include/chain.h
CHAIN_ACTS = {"relu": 0, "gelu": 1, "silu": 2, "gelu_tanh": 3}


def _check_chain(x, b):
    import torch
    for name, t in (("x", x), ("b", b)):
        if not isinstance(t, torch.Tensor) or not t.is_cuda or t.dtype != torch.bfloat16 or \
                not t.is_contiguous():
            raise TypeError(f"{name} must be a contiguous CUDA bf16 tensor")
    if x.dim() != 2 or b.dim() != 1 or b.shape[0] != x.shape[1]:
        raise ValueError("x [rows, cols] and b [cols] expected")
    return int(x.shape[0]), int(x.shape[1])


def chain_fused(x, b, y=None, alpha=1.0, act="gelu", stream=None):
    """y = act(alpha * x + b) in one kernel (bf16 in and out)."""
    import torch
    rows, cols = _check_chain(x, b)
    y = torch.empty_like(x) if y is None else y
    st = abi.chain_fused(x.data_ptr(), b.data_ptr(), y.data_ptr(), rows, cols, float(alpha),
                         CHAIN_ACTS[act], _stream_handle(stream))
    if st != ATTN_OK:
        raise AttnError(st, "chain_fused")
    return y


def chain_unfused(x, b, y=None, tmp=None, alpha=1.0, act="gelu", stream=None):
    """The same chain as three kernels through a bf16 scratch tensor."""
    import torch
    rows, cols = _check_chain(x, b)
    y = torch.empty_like(x) if y is None else y
    tmp = torch.empty_like(x) if tmp is None else tmp
    st = abi.chain_unfused(x.data_ptr(), b.data_ptr(), y.data_ptr(), tmp.data_ptr(), rows, cols,
                           float(alpha), CHAIN_ACTS[act], _stream_handle(stream))
    if st != ATTN_OK:
        raise AttnError(st, "chain_unfused")
    return y


def naive_workspace_bytes(B: int, H: int, N: int) -> int:
    return abi.attn_fwd_naive_workspace_bytes(B, H, N)


def attn_fwd_naive(q, k, v, o=None, lse=None, scale=None, causal=False, workspace=None,
                   stream=None):
    """Unfused three-kernel forward (S and P in HBM). Returns (o, lse)."""
    import torch
    B, H, N, d = _check_qkv(q, k, v)
    o, lse = _outputs(q, o, lse)
    need = naive_workspace_bytes(B, H, N)
    if workspace is None:
        workspace = torch.empty((need,), dtype=torch.uint8, device=q.device)
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    st = abi.attn_fwd_naive(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                            lse.data_ptr(), B, H, N, d, scale, int(bool(causal)),
                            workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                            _stream_handle(stream))
    if st != ATTN_OK:
        raise AttnError(st, "attn_fwd_naive")
    return o, lse


def last_device_error(stream=None) -> int:
    """Reads and clears the device error word (synchronises the stream)."""
    return abi.attn_last_device_error(_stream_handle(stream))


def selftest_wait_timeout(limit_ms: int, stream=None) -> int:
    return abi.attn_selftest_wait_timeout(int(limit_ms), _stream_handle(stream))


def set_wait_limit_ms(ms: int) -> None:
    """Limit of every bounded wait in the kernels launched from now on."""
    st = abi.attn_set_wait_limit_ms(int(ms))
    if st != ATTN_OK:
        raise AttnError(st, "attn_set_wait_limit_ms")


def wait_limit_ms() -> int:
    return abi.attn_wait_limit_ms()
