"""ctypes binding of ``libllmint8.so`` (the C ABI in ``include/llmint8.h``).

Argument marshalling only: tensors are checked for dtype/device/layout and
their device pointers, sizes and the current CUDA stream are passed to the C
functions, which run every step of the method in CUDA kernels.  There is no
CPU fallback: if the library is missing or fails to load, every call raises.
"""
from __future__ import annotations

import ctypes
import os
import re
import threading
from typing import Dict, Optional, Tuple

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libllmint8.so")
HEADER = os.path.join(os.path.dirname(PKG), "include", "llmint8.h")

STATUS_NAMES = {
    0: "LLMINT8_OK",
    1: "LLMINT8_ERR_INVALID_ARG",
    2: "LLMINT8_ERR_UNSUPPORTED",
    3: "LLMINT8_ERR_WORKSPACE",
    4: "LLMINT8_ERR_CUDA",
    5: "LLMINT8_ERR_OUTLIER_OVERFLOW",
    6: "LLMINT8_ERR_TIMEOUT",
}
OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_WORKSPACE, ERR_CUDA, ERR_OUTLIER_OVERFLOW, ERR_TIMEOUT = range(7)
STATUS_OUTLIER_OVERFLOW = 0x1
STATUS_TIMEOUT = 0x2


class LLMInt8Error(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}")


class WsLayout(ctypes.Structure):
    _fields_ = [
        ("status", ctypes.c_size_t),
        ("n_outlier", ctypes.c_size_t),
        ("outlier_idx", ctypes.c_size_t),
        ("row_scale", ctypes.c_size_t),
        ("xq", ctypes.c_size_t),
        ("xo", ctypes.c_size_t),
        ("ldq", ctypes.c_int64),
        ("ldo", ctypes.c_int64),
        ("total", ctypes.c_size_t),
    ]


_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_F = ctypes.c_float
_SZ = ctypes.c_size_t
_ST = ctypes.c_int

SIGNATURES = {
    "llmint8_status_string": (ctypes.c_char_p, [_ST]),
    "llmint8_workspace_size": (_SZ, [_I64, _I64, _I64, _I64]),
    "llmint8_workspace_init": (_ST, [_P, _SZ, _P]),
    "llmint8_workspace_layout": (_ST, [_I64, _I64, _I64, _I64, ctypes.POINTER(WsLayout)]),
    "llmint8_quantize_weight_colwise": (_ST, [_P, _I64, _I64, _I64, _P, _I64, _P, _P]),
    "llmint8_quantize_act_rowwise_outliers": (_ST, [_P, _I64, _I64, _I64, _F, _P, _I64, _P, _P, _I64, _P, _P,
                                                    _I64, _P, _SZ, _P]),
    "llmint8_mixed_matmul": (_ST, [_P, _I64, _I64, _I64, _P, _I64, _P, _P, _I64, _P, _I64, _F, _I64, _P, _I64,
                                   _P, _SZ, _P]),
    "llmint8_mixed_gemm": (_ST, [_P, _I64, _P, _P, _P, _I64, _P, _I64, _P, _I64, _P, _P, _I64, _P, _I64, _I64,
                                 _I64, _P, _I64, _P, _SZ, _P]),
    "llmint8_quantize_act_rowwise_outliers_noalloc": (_ST, [_P, _I64, _I64, _I64, _F, _P, _I64, _P, _P, _I64, _P,
                                                            _P, _I64, _P]),
    "llmint8_check_status": (_ST, [_P, _P, ctypes.POINTER(ctypes.c_uint32)]),
    "llmint8_mixed_matmul_kernels": (ctypes.c_int, [_I64, _I64, _I64, _I64, _P]),
    "llmint8_mixed_matmul_path": (ctypes.c_char_p, [_I64, _I64, _I64, _I64, _I64, _P]),
    "llmint8_outlier_stats": (_ST, [_P, _I64, _I64, _I64, _F, _P, _P, _SZ, _P]),
    "llmint8_debug_int8_gemm_i32": (_ST, [_P, _I64, _P, _I64, _I64, _I64, _I64, _P, _I64, _P, _SZ, _P]),
    "llmint8_debug_mixed_matmul_i32": (_ST, [_P, _I64, _I64, _I64, _P, _I64, _P, _I64, _F, _I64, _P, _I64, _P,
                                             _SZ, _P]),
    "llmint8_debug_set_waits": (_ST, [ctypes.c_uint64, ctypes.c_uint32]),
    "llmint8_unshard_columns": (_ST, [_P, _I64, _I64, _I64, _P, _P, _I64, _P]),
}

_lock = threading.Lock()
_lib = None


def lib() -> ctypes.CDLL:
    """Load the in-tree library (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                                   "`python -m int8_quantized_matmul_colwise_b200._build`")
            L = ctypes.CDLL(LIB_PATH)
            for name, (res, args) in SIGNATURES.items():
                fn = getattr(L, name)
                fn.restype = res
                fn.argtypes = args
            _lib = L
        return _lib


def header_functions():
    """Names of the functions include/llmint8.h declares."""
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(llmint8_[a-z0-9_]+)\s*\(", text)))


def _check(status: int, where: str):
    if status != OK:
        raise LLMInt8Error(status, where)


# ------------------------------------------------------------------ torch marshalling
def _torch():
    import torch
    return torch


def _stream(stream=None) -> int:
    torch = _torch()
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _rowmajor(t, name: str, dtype, ndim=2):
    torch = _torch()
    if t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name}: must be a CUDA tensor")
    if t.dim() != ndim:
        raise ValueError(f"{name}: expected {ndim} dims, got {t.dim()}")
    if ndim == 2 and t.stride(1) != 1:
        raise ValueError(f"{name}: inner dimension must be contiguous")
    if ndim == 1 and t.stride(0) != 1:
        raise ValueError(f"{name}: must be contiguous")
    return t


def _vector(t, name: str, n: int):
    """An optional fp16 [n] device vector (the linear layer's bias)."""
    if t is None:
        return None
    torch = _torch()
    _rowmajor(t, name, torch.float16, 1)
    if t.numel() != n:
        raise ValueError(f"{name}: expected {n} elements, got {t.numel()}")
    return t


def _ld(t) -> int:
    return t.stride(0) if t.size(0) > 1 else max(t.stride(0), t.size(1))


def round_up(v: int, m: int) -> int:
    return (v + m - 1) // m * m


# ------------------------------------------------------------------ same names as the C ABI
def llmint8_status_string(status: int) -> str:
    return lib().llmint8_status_string(status).decode()


def llmint8_workspace_size(M: int, N: int, K: int, outlier_cap: int) -> int:
    return int(lib().llmint8_workspace_size(M, N, K, outlier_cap))


def llmint8_workspace_layout(M: int, N: int, K: int, outlier_cap: int) -> WsLayout:
    L = WsLayout()
    _check(lib().llmint8_workspace_layout(M, N, K, outlier_cap, ctypes.byref(L)), "llmint8_workspace_layout")
    return L


def llmint8_workspace_init(ws, stream=None):
    _check(lib().llmint8_workspace_init(_ptr(ws), ws.numel() * ws.element_size(), _stream(stream)),
           "llmint8_workspace_init")


def llmint8_quantize_weight_colwise(W, Wq, col_scale, stream=None):
    """W fp16 [K, N] -> Wq int8 [N, ldk] (K contiguous), col_scale fp32 [N]."""
    torch = _torch()
    _rowmajor(W, "W", torch.float16)
    _rowmajor(Wq, "Wq", torch.int8)
    _rowmajor(col_scale, "col_scale", torch.float32, 1)
    K, N = W.shape
    if Wq.size(0) != N or Wq.size(1) < K or col_scale.numel() != N:
        raise ValueError("Wq must be [N, >=K] and col_scale [N]")
    _check(lib().llmint8_quantize_weight_colwise(_ptr(W), K, N, _ld(W), _ptr(Wq), _ld(Wq), _ptr(col_scale),
                                                 _stream(stream)), "llmint8_quantize_weight_colwise")


def llmint8_quantize_act_rowwise_outliers(X, tau: float, Xq, row_scale, outlier_idx, n_outlier, Xo, ws,
                                          stream=None):
    torch = _torch()
    _rowmajor(X, "X", torch.float16)
    _rowmajor(Xq, "Xq", torch.int8)
    _rowmajor(row_scale, "row_scale", torch.float32, 1)
    _rowmajor(outlier_idx, "outlier_idx", torch.int32, 1)
    _rowmajor(n_outlier, "n_outlier", torch.int32, 1)
    M, K = X.shape
    ldo = 0
    if Xo is not None:
        _rowmajor(Xo, "Xo", torch.float16)
        ldo = _ld(Xo)
    _check(lib().llmint8_quantize_act_rowwise_outliers(
        _ptr(X), M, K, _ld(X), float(tau), _ptr(Xq), _ld(Xq), _ptr(row_scale), _ptr(outlier_idx),
        outlier_idx.numel(), _ptr(n_outlier), _ptr(Xo), ldo, _ptr(ws), ws.numel() * ws.element_size(),
        _stream(stream)), "llmint8_quantize_act_rowwise_outliers")


def llmint8_mixed_matmul(X, Wq, col_scale, W, tau: float, outlier_cap: int, Y, ws, stream=None, bias=None):
    torch = _torch()
    _rowmajor(X, "X", torch.float16)
    _rowmajor(Wq, "Wq", torch.int8)
    _rowmajor(col_scale, "col_scale", torch.float32, 1)
    if W is not None:  # None: no fp16 weight kept, the outlier rows come from Wq
        _rowmajor(W, "W", torch.float16)
    _rowmajor(Y, "Y", torch.float16)
    M, K = X.shape
    N = Wq.size(0)
    _check(lib().llmint8_mixed_matmul(
        _ptr(X), M, K, _ld(X), _ptr(Wq), _ld(Wq), _ptr(col_scale), _ptr(W), 0 if W is None else _ld(W),
        _ptr(_vector(bias, "bias", N)), N, float(tau),
        int(outlier_cap), _ptr(Y), _ld(Y), _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)),
        "llmint8_mixed_matmul")


def llmint8_mixed_gemm(Xq, row_scale, outlier_idx, n_outlier, Xo, Wq, col_scale, W, K: int, Y, ws,
                       stream=None, bias=None):
    torch = _torch()
    _rowmajor(Xq, "Xq", torch.int8)
    _rowmajor(row_scale, "row_scale", torch.float32, 1)
    _rowmajor(outlier_idx, "outlier_idx", torch.int32, 1)
    _rowmajor(n_outlier, "n_outlier", torch.int32, 1)
    _rowmajor(Xo, "Xo", torch.float16)
    _rowmajor(Wq, "Wq", torch.int8)
    _rowmajor(col_scale, "col_scale", torch.float32, 1)
    if W is not None:  # None: no fp16 weight kept, the outlier rows come from Wq
        _rowmajor(W, "W", torch.float16)
    _rowmajor(Y, "Y", torch.float16)
    M, N = Xq.size(0), Wq.size(0)
    _check(lib().llmint8_mixed_gemm(
        _ptr(Xq), _ld(Xq), _ptr(row_scale), _ptr(outlier_idx), _ptr(n_outlier), outlier_idx.numel(), _ptr(Xo),
        _ld(Xo), _ptr(Wq), _ld(Wq), _ptr(col_scale), _ptr(W), 0 if W is None else _ld(W),
        _ptr(_vector(bias, "bias", Wq.size(0))), M, N, K, _ptr(Y), _ld(Y),
        _ptr(ws),
        ws.numel() * ws.element_size(), _stream(stream)), "llmint8_mixed_gemm")


def llmint8_check_status(ws, stream=None) -> Tuple[int, int]:
    """(status, raw flags); synchronises the stream and clears the word."""
    flags = ctypes.c_uint32(0)
    st = lib().llmint8_check_status(_ptr(ws), _stream(stream), ctypes.byref(flags))
    return int(st), int(flags.value)


def llmint8_outlier_stats(X, tau: float, stats, ws, stream=None):
    """stats int64 [3] (device) <- values with |x| >= tau, their columns, their rows."""
    torch = _torch()
    _rowmajor(X, "X", torch.float16)
    _rowmajor(stats, "stats", torch.int64, 1)
    if stats.numel() != 3:
        raise ValueError("stats: expected 3 elements")
    M, K = X.shape
    _check(lib().llmint8_outlier_stats(_ptr(X), M, K, _ld(X), float(tau), _ptr(stats), _ptr(ws),
                                       ws.numel() * ws.element_size(), _stream(stream)), "llmint8_outlier_stats")


def llmint8_mixed_matmul_kernels(X, N: int) -> int:
    """Kernels llmint8_mixed_matmul launches for this X and N (1, 2 or 3)."""
    M, K = X.shape
    return int(lib().llmint8_mixed_matmul_kernels(M, N, K, _ld(X), _ptr(X)))


def llmint8_mixed_matmul_path(X, Wq, K: int):
    """Names of the kernels llmint8_mixed_matmul launches for this X and Wq
    ([N, ldk] int8), in launch order; None if the call would be rejected."""
    M = X.shape[0]
    N = Wq.shape[0]
    r = lib().llmint8_mixed_matmul_path(M, N, K, _ld(X), _ld(Wq), _ptr(X))
    return None if r is None else r.decode().split(",")


def llmint8_debug_int8_gemm_i32(Xq, Wq, K: int, C, ws, stream=None):
    torch = _torch()
    _rowmajor(Xq, "Xq", torch.int8)
    _rowmajor(Wq, "Wq", torch.int8)
    _rowmajor(C, "C", torch.int32)
    M, N = Xq.size(0), Wq.size(0)
    _check(lib().llmint8_debug_int8_gemm_i32(_ptr(Xq), _ld(Xq), _ptr(Wq), _ld(Wq), M, N, K, _ptr(C), _ld(C),
                                             _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)),
           "llmint8_debug_int8_gemm_i32")


def llmint8_debug_mixed_matmul_i32(X, Wq, col_scale, tau: float, outlier_cap: int, C, ws, stream=None):
    """Test hook: the path of llmint8_mixed_matmul with the raw int32
    accumulator stored in C [M, >= N] instead of Y."""
    torch = _torch()
    _rowmajor(X, "X", torch.float16)
    _rowmajor(Wq, "Wq", torch.int8)
    _rowmajor(col_scale, "col_scale", torch.float32, 1)
    _rowmajor(C, "C", torch.int32)
    M, K = X.shape
    N = Wq.size(0)
    _check(lib().llmint8_debug_mixed_matmul_i32(
        _ptr(X), M, K, _ld(X), _ptr(Wq), _ld(Wq), _ptr(col_scale), N, float(tau), int(outlier_cap), _ptr(C), _ld(C),
        _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)), "llmint8_debug_mixed_matmul_i32")


DEFAULT_WAIT_LIMIT_NS = 2_000_000_000
STALL_ACT_GRID_BARRIER = 0x1
STALL_GEMV_WEIGHT = 0x2
STALL_GEMM_OPERANDS = 0x4


def llmint8_debug_set_waits(limit_ns: int = DEFAULT_WAIT_LIMIT_NS, stall_mask: int = 0):
    """Test hook: the bound of the kernels' bounded waits and the mask of
    waits held back (see include/llmint8.h).  Defaults restore normal use."""
    _check(lib().llmint8_debug_set_waits(int(limit_ns), int(stall_mask)), "llmint8_debug_set_waits")


# ------------------------------------------------------------------ allocation helpers (torch memory)
def empty_workspace(M: int, N: int, K: int, outlier_cap: int, device="cuda"):
    """A zero-filled workspace tensor (uint8) sized for these sizes."""
    torch = _torch()
    size = llmint8_workspace_size(M, N, K, outlier_cap)
    if size == 0:
        raise LLMInt8Error(ERR_INVALID_ARG, "llmint8_workspace_size")
    return torch.zeros(size, dtype=torch.uint8, device=device)


def workspace_views(ws, M: int, N: int, K: int, outlier_cap: int) -> Dict[str, object]:
    """Views of the intermediates a mixed-matmul call leaves in its workspace."""
    torch = _torch()
    L = llmint8_workspace_layout(M, N, K, outlier_cap)
    b = ws
    return {
        "status": b[L.status:L.status + 4].view(torch.int32),
        "n_outlier": b[L.n_outlier:L.n_outlier + 4].view(torch.int32),
        "outlier_idx": b[L.outlier_idx:L.outlier_idx + 4 * outlier_cap].view(torch.int32),
        "row_scale": b[L.row_scale:L.row_scale + 4 * M].view(torch.float32),
        "xq": b[L.xq:L.xq + M * L.ldq].view(torch.int8).view(M, L.ldq),
        "xo": b[L.xo:L.xo + 2 * M * L.ldo].view(torch.float16).view(M, L.ldo),
    }
