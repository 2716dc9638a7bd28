"""LLM.int8() mixed-precision decomposition matmul for NVIDIA B200 (sm_100a).

Y = X . W with the outlier feature dimensions of X (any |x| >= tau) multiplied
in 16-bit and everything else in int8 with one absmax scale per row of X and
per column of W ("LLM.int8(): 8-bit Matrix Multiplication for Transformers at
Scale", arXiv abstract; "Compress your LLMs", Vector-wise quantization and
Mixed-precision decomposition).

The work runs in hand-written CUDA kernels behind the C ABI of
``include/llmint8.h`` (``libllmint8.so``, built in-tree); this package only
marshals torch tensors to it (``capi``) and offers allocating conveniences.
"""
from __future__ import annotations

from typing import Dict, Optional, Tuple

from . import capi
from .capi import (LLMInt8Error, empty_workspace, llmint8_check_status, llmint8_debug_int8_gemm_i32,
                   llmint8_debug_mixed_matmul_i32, llmint8_debug_set_waits,
                   llmint8_mixed_gemm, llmint8_mixed_matmul, llmint8_mixed_matmul_kernels, llmint8_mixed_matmul_path,
                   llmint8_outlier_stats,
                   llmint8_quantize_act_rowwise_outliers, llmint8_quantize_weight_colwise,
                   llmint8_status_string, llmint8_workspace_init, llmint8_workspace_layout,
                   llmint8_workspace_size, round_up, workspace_views)

__all__ = [
    "capi", "LLMInt8Error", "quantize_weight_colwise", "quantize_act_rowwise_outliers", "mixed_matmul",
    "check_status", "debug_int8_gemm_i32", "empty_workspace", "workspace_views", "Int8Weight",
    "llmint8_quantize_weight_colwise", "llmint8_quantize_act_rowwise_outliers", "llmint8_mixed_matmul",
    "llmint8_mixed_gemm", "mixed_gemm",
    "llmint8_check_status", "llmint8_debug_int8_gemm_i32", "llmint8_status_string", "llmint8_workspace_size",
    "llmint8_workspace_init", "llmint8_workspace_layout", "llmint8_mixed_matmul_kernels",
    "llmint8_mixed_matmul_path",
    "llmint8_outlier_stats", "outlier_stats", "Int8Linear", "llmint8_debug_mixed_matmul_i32",
    "llmint8_debug_set_waits", "debug_mixed_matmul_i32",
]


def quantize_weight_colwise(W, stream=None):
    """W fp16 [K, N] -> (Wq int8 [N, round_up(K,16)], col_scale fp32 [N])."""
    import torch
    K, N = W.shape
    Wq = torch.empty((N, round_up(K, 16)), dtype=torch.int8, device=W.device)
    cs = torch.empty(N, dtype=torch.float32, device=W.device)
    llmint8_quantize_weight_colwise(W, Wq, cs, stream)
    return Wq, cs


def quantize_act_rowwise_outliers(X, tau: float = 6.0, outlier_cap: Optional[int] = None, ws=None,
                                  stream=None) -> Dict[str, object]:
    """Steps a1-a4 on X fp16 [M, K]; returns device tensors Xq, row_scale,
    outlier_idx (first min(n_o, cap) valid), n_outlier [1] and Xo."""
    import torch
    M, K = X.shape
    cap = K if outlier_cap is None else outlier_cap
    dev = X.device
    out = {
        "Xq": torch.empty((M, round_up(K, 16)), dtype=torch.int8, device=dev),
        "row_scale": torch.empty(M, dtype=torch.float32, device=dev),
        "outlier_idx": torch.empty(cap, dtype=torch.int32, device=dev),
        "n_outlier": torch.empty(1, dtype=torch.int32, device=dev),
        "Xo": torch.empty((M, cap), dtype=torch.float16, device=dev),
    }
    if ws is None:
        ws = empty_workspace(M, 1, K, cap, device=dev)
    llmint8_quantize_act_rowwise_outliers(X, tau, out["Xq"], out["row_scale"], out["outlier_idx"],
                                          out["n_outlier"], out["Xo"], ws, stream)
    out["ws"] = ws
    out["K"] = K
    return out


def mixed_matmul(X, Wq, col_scale, W, tau: float = 6.0, outlier_cap: Optional[int] = None, Y=None, ws=None,
                 stream=None, bias=None):
    """Y = X . W (+ bias) by the LLM.int8() decomposition (fp16 [M, N]).
    W = None: no fp16 weight kept, the outlier rows are recovered from Wq."""
    import torch
    M, K = X.shape
    N = Wq.size(0)
    cap = K if outlier_cap is None else outlier_cap
    if Y is None:
        Y = torch.empty((M, N), dtype=torch.float16, device=X.device)
    if ws is None:
        ws = empty_workspace(M, N, K, cap, device=X.device)
    llmint8_mixed_matmul(X, Wq, col_scale, W, tau, cap, Y, ws, stream, bias)
    return Y


def mixed_gemm(act: Dict[str, object], Wq, col_scale, W, Y=None, ws=None, stream=None, bias=None):
    """Steps a5-a7 on the output of quantize_act_rowwise_outliers."""
    import torch
    Xq = act["Xq"]
    M, N = Xq.size(0), Wq.size(0)
    K = W.size(0) if W is not None else int(act["K"])  # W None: int8-only weight
    if Y is None:
        Y = torch.empty((M, N), dtype=torch.float16, device=Xq.device)
    if ws is None:
        ws = act["ws"]
    llmint8_mixed_gemm(Xq, act["row_scale"], act["outlier_idx"], act["n_outlier"], act["Xo"], Wq, col_scale, W,
                       K, Y, ws, stream, bias)
    return Y


def outlier_stats(X, tau: float = 6.0, ws=None, stream=None) -> Dict[str, int]:
    """Values with |x| >= tau in X, the feature columns and the rows holding
    them (reads the three counts back to the host)."""
    import torch
    M, K = X.shape
    if ws is None:
        ws = empty_workspace(1, 1, K, K, device=X.device)
    stats = torch.empty(3, dtype=torch.int64, device=X.device)
    llmint8_outlier_stats(X, tau, stats, ws, stream)
    v = stats.tolist()
    return {"values": int(v[0]), "columns": int(v[1]), "rows": int(v[2])}


def check_status(ws, stream=None) -> int:
    """Raise if the device reported an outlier overflow or a timeout."""
    st, _ = llmint8_check_status(ws, stream)
    if st != capi.OK:
        raise LLMInt8Error(st, "device status")
    return st


def debug_int8_gemm_i32(Xq, Wq, K: int, stream=None):
    """int32 [M, N] = Xq[:, :K] . Wq[:, :K]^T through the tcgen05 kernel."""
    import torch
    M, N = Xq.size(0), Wq.size(0)
    C = torch.empty((M, N), dtype=torch.int32, device=Xq.device)
    ws = empty_workspace(M, N, K, 1, device=Xq.device)  # status word + decode split-K scratch
    llmint8_debug_int8_gemm_i32(Xq, Wq, K, C, ws, stream)
    return C


def debug_mixed_matmul_i32(X, Wq, col_scale, tau: float = 6.0, outlier_cap: Optional[int] = None, ws=None,
                           stream=None):
    """int32 [M, N]: the accumulator the whole path computes for X (same
    kernels as mixed_matmul), and the workspace holding its Xq, rs, O, Xo."""
    import torch
    M, K = X.shape
    N = Wq.size(0)
    cap = K if outlier_cap is None else outlier_cap
    C = torch.empty((M, N), dtype=torch.int32, device=X.device)
    if ws is None:
        ws = empty_workspace(M, N, K, cap, device=X.device)
    llmint8_debug_mixed_matmul_i32(X, Wq, col_scale, tau, cap, C, ws, stream)
    return C, ws


class Int8Weight:
    """A weight converted once at load time: int8 codes, column scales and
    the fp16 matrix whose outlier rows the 16-bit product reads."""

    def __init__(self, W, stream=None):
        self.W = W
        self.K, self.N = W.shape
        self.Wq, self.col_scale = quantize_weight_colwise(W, stream)

    def matmul(self, X, tau: float = 6.0, outlier_cap: Optional[int] = None, Y=None, ws=None, stream=None):
        return mixed_matmul(X, self.Wq, self.col_scale, self.W, tau, outlier_cap, Y, ws, stream)


def __getattr__(name):
    # the torch module wrapper is imported on first use
    if name == "Int8Linear":
        from .linear import Int8Linear
        return Int8Linear
    raise AttributeError(name)
