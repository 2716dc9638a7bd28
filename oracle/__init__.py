"""CPU oracle for the LLM.int8() mixed-precision decomposition matmul.

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the benchmark's CPU
baseline call it; the product path never imports it.  The arithmetic lives in
plain C (``llmint8_oracle.c``); this module builds that file with gcc and
marshals numpy arrays to it.  It shares no code with the CUDA library.

Every function follows the pages (titles and sections are cited in the C file):
outlier columns (a1), row scales (a2), row quantization (a3), column-wise weight
quantization (a0), outlier gather (a4), int8 matmul (a5), dequantize + 16-bit
outlier product + fp16 output (a6, a7).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from typing import Dict, Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "llmint8_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_CFLAGS = ["-O2", "-std=c11", "-fopenmp", "-fno-fast-math", "-ffp-contract=off", "-fPIC", "-shared"]
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle into ``oracle/liboracle.so`` (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *_CFLAGS, _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        path = os.environ.get("LLMINT8_ORACLE_LIB")  # a mutant build, used by the pin-strength test
        if not path:
            path = build()
        lib = ctypes.CDLL(path)
        P = ctypes.c_void_p
        I64 = ctypes.c_int64
        F = ctypes.c_float
        sig = {
            "oracle_half_to_double_array": (None, [P, I64, P]),
            "oracle_double_to_half_array": (None, [P, I64, P]),
            "oracle_quantize_value": (ctypes.c_int8, [F, F]),
            "oracle_outlier_columns": (I64, [P, I64, I64, I64, F, P]),
            "oracle_row_scales": (None, [P, I64, I64, I64, P, I64, P]),
            "oracle_quantize_rows": (None, [P, I64, I64, I64, P, I64, P, P]),
            "oracle_col_scales": (None, [P, I64, I64, P]),
            "oracle_quantize_cols": (None, [P, I64, I64, P, P]),
            "oracle_gather_outliers": (None, [P, I64, I64, P, I64, P, P, I64, P]),
            "oracle_int8_matmul": (None, [P, P, I64, I64, P, I64, P]),
            "oracle_mixed_output": (None, [P, P, P, P, I64, P, I64, P, I64, P, P, I64, P, P]),
            "oracle_dequantize_weight": (None, [P, I64, I64, P, P]),
            "oracle_outlier_stats": (None, [P, I64, I64, I64, ctypes.c_float, P]),
            "oracle_num_threads": (ctypes.c_int, []),
        }
        for name, (res, args) in sig.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
        return lib


def _p(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data


def _c(a: np.ndarray, dtype) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=dtype)


def _bits16(a: np.ndarray) -> np.ndarray:
    a = np.ascontiguousarray(a)
    if a.dtype == np.float16:
        return a.view(np.uint16)
    assert a.dtype == np.uint16, a.dtype
    return a


# ---------------------------------------------------------------- codec

def half_to_double(h: np.ndarray) -> np.ndarray:
    h = _bits16(h).ravel()
    out = np.empty(h.size, np.float64)
    _load().oracle_half_to_double_array(_p(h), h.size, _p(out))
    return out


def double_to_half(v: np.ndarray) -> np.ndarray:
    v = _c(v, np.float64).ravel()
    out = np.empty(v.size, np.uint16)
    _load().oracle_double_to_half_array(_p(v), v.size, _p(out))
    return out.view(np.float16)


def quantize_value(x: float, s: float) -> int:
    return int(_load().oracle_quantize_value(float(x), float(s)))


# ---------------------------------------------------------------- method steps

def outlier_columns(X: np.ndarray, tau: float) -> np.ndarray:
    """a1: ascending int32 array of columns with some |x| >= tau."""
    Xb = _bits16(X)
    M, K = Xb.shape
    O = np.empty(max(K, 1), np.int32)
    n = _load().oracle_outlier_columns(_p(Xb), M, K, K, float(tau), _p(O))
    return O[:n].copy()


def row_scales(X: np.ndarray, O: np.ndarray) -> np.ndarray:
    """a2: fp32 [M] absmax of each row over the non-outlier columns."""
    Xb = _bits16(X)
    M, K = Xb.shape
    O = _c(O, np.int32)
    rs = np.empty(M, np.float32)
    _load().oracle_row_scales(_p(Xb), M, K, K, _p(O), O.size, _p(rs))
    return rs


def quantize_rows(X: np.ndarray, O: np.ndarray, rs: np.ndarray) -> np.ndarray:
    """a3: int8 [M, K]; outlier columns are zero."""
    Xb = _bits16(X)
    M, K = Xb.shape
    O = _c(O, np.int32)
    rs = _c(rs, np.float32)
    Xq = np.empty((M, K), np.int8)
    _load().oracle_quantize_rows(_p(Xb), M, K, K, _p(O), O.size, _p(rs), _p(Xq))
    return Xq


def col_scales(W: np.ndarray) -> np.ndarray:
    """a0: fp32 [N] absmax of each column of W over all K rows."""
    Wb = _bits16(W)
    K, N = Wb.shape
    cs = np.empty(N, np.float32)
    _load().oracle_col_scales(_p(Wb), K, N, _p(cs))
    return cs


def quantize_cols(W: np.ndarray, cs: np.ndarray) -> np.ndarray:
    """a0: int8 [K, N] (W's own layout)."""
    Wb = _bits16(W)
    K, N = Wb.shape
    cs = _c(cs, np.float32)
    Wq = np.empty((K, N), np.int8)
    _load().oracle_quantize_cols(_p(Wb), K, N, _p(cs), _p(Wq))
    return Wq


def gather_outliers(X: np.ndarray, O: np.ndarray, W: Optional[np.ndarray] = None):
    """a4: Xo = X[:, O] (fp16 [M, n_o]) and, if W is given, Wo = W[O, :]."""
    Xb = _bits16(X)
    M, K = Xb.shape
    O = _c(O, np.int32)
    Xo = np.empty((M, O.size), np.uint16)
    Wb = None if W is None else _bits16(W)
    N = 0 if W is None else Wb.shape[1]
    Wo = None if W is None else np.empty((O.size, N), np.uint16)
    _load().oracle_gather_outliers(_p(Xb), M, K, _p(O), O.size, _p(Xo), _p(Wb), N, _p(Wo))
    return Xo.view(np.float16), (None if Wo is None else Wo.view(np.float16))


def int8_matmul(Xq: np.ndarray, Wq: np.ndarray, rows: Optional[np.ndarray] = None) -> np.ndarray:
    """a5: int64 [len(rows) or M, N] = Xq[rows] . Wq (Wq in [K, N] layout)."""
    Xq = _c(Xq, np.int8)
    Wq = _c(Wq, np.int8)
    M, K = Xq.shape
    K2, N = Wq.shape
    assert K == K2
    rr = None if rows is None else _c(rows, np.int64)
    n = M if rr is None else rr.size
    acc = np.empty((n, N), np.int64)
    _load().oracle_int8_matmul(_p(Xq), _p(Wq), N, K, _p(rr), n, _p(acc))
    return acc


def mixed_output(acc: np.ndarray, rs: np.ndarray, cs: np.ndarray, X: np.ndarray, W: np.ndarray,
                 O: np.ndarray, rows: Optional[np.ndarray] = None, bias: Optional[np.ndarray] = None):
    """a6+a7: (Y fp16, Yd float64) for the selected rows; optional fp16 bias [N]."""
    acc = _c(acc, np.int64)
    Xb = _bits16(X)
    Wb = _bits16(W)
    M, K = Xb.shape
    N = Wb.shape[1]
    O = _c(O, np.int32)
    rr = None if rows is None else _c(rows, np.int64)
    n = M if rr is None else rr.size
    assert acc.shape == (n, N)
    Yd = np.empty((n, N), np.float64)
    Y = np.empty((n, N), np.uint16)
    bb = None if bias is None else _bits16(np.asarray(bias, np.float16).reshape(N))
    _load().oracle_mixed_output(_p(acc), _p(_c(rs, np.float32)), _p(_c(cs, np.float32)), _p(Xb), K,
                                _p(Wb), N, _p(O), O.size, _p(bb), _p(rr), n, _p(Yd), _p(Y))
    return Y.view(np.float16), Yd


def outlier_stats(X: np.ndarray, tau: float) -> Dict[str, int]:
    """Outlier values (|x| >= tau), their feature columns and their rows."""
    Xb = _bits16(X)
    M, K = Xb.shape
    out = np.zeros(3, np.int64)
    _load().oracle_outlier_stats(_p(Xb), M, K, K, ctypes.c_float(tau), _p(out))
    return {"values": int(out[0]), "columns": int(out[1]), "rows": int(out[2])}


def dequantize_weight(Wq: np.ndarray, cs: np.ndarray) -> np.ndarray:
    """fp16 [K, N]: the weight recovered from its int8 form, Wq * cs / 127
    rounded once to fp16 (the outlier rows when no fp16 weight is kept)."""
    Wq = _c(Wq, np.int8)
    K, N = Wq.shape
    out = np.empty((K, N), np.uint16)
    _load().oracle_dequantize_weight(_p(Wq), K, N, _p(_c(cs, np.float32)), _p(out))
    return out.view(np.float16)


def quantize_weight(W: np.ndarray):
    """a0 as one call: (Wq [K, N] int8, cs [N] fp32)."""
    cs = col_scales(W)
    return quantize_cols(W, cs), cs


def quantize_activation(X: np.ndarray, tau: float):
    """a1-a3 as one call: (O, rs, Xq)."""
    O = outlier_columns(X, tau)
    rs = row_scales(X, O)
    return O, rs, quantize_rows(X, O, rs)


def mixed_matmul(X: np.ndarray, W: np.ndarray, tau: float, rows: Optional[np.ndarray] = None,
                 weight: Optional[tuple] = None, int8_weight: bool = False,
                 bias: Optional[np.ndarray] = None) -> Dict[str, np.ndarray]:
    """The whole path a0..a7; returns every intermediate.

    ``rows`` restricts a5-a7 to those rows (a1 still scans all rows, as the
    definition requires).  ``weight`` may pass a precomputed (Wq, cs).
    ``int8_weight``: the outlier product uses the weight recovered from its
    int8 form (dequantize_weight) instead of the fp16 W.  ``bias``: fp16 [N]
    added to every row (a linear layer's X W + b)."""
    Wq, cs = quantize_weight(W) if weight is None else weight
    O, rs, Xq = quantize_activation(X, tau)
    acc = int8_matmul(Xq, Wq, rows)
    Wout = dequantize_weight(Wq, cs) if int8_weight else W
    Y, Yd = mixed_output(acc, rs, cs, X, Wout, O, rows, bias)
    return {"O": O, "rs": rs, "Xq": Xq, "Wq": Wq, "cs": cs, "acc": acc, "Y": Y, "Yd": Yd}


def num_threads() -> int:
    return int(_load().oracle_num_threads())
