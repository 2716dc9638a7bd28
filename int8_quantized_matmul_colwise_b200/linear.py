"""A linear layer y = x W^T + b computed by the LLM.int8() decomposition.

The method is a drop-in for the transformer's feed-forward and attention
projection layers: a 16-bit checkpoint is loaded, converted to int8 once and
used at once ("LLM.int8(): 8-bit Matrix Multiplication for Transformers at
Scale", arXiv abstract; "8-bit Matrix Multiplication for Large Language
Models", Summary & Methodology Analysis).  This module does the conversion at
construction (column-wise int8 weight + column scales) and runs every forward
through the C ABI (``llmint8_mixed_matmul``): activation outliers, row-wise
quantization, the tcgen05 int8 GEMM, the 16-bit outlier product and the bias,
all in the library's kernels.  There is no CPU path: inputs must be fp16 CUDA
tensors.

By default the fp16 weight is not kept (the outlier rows are recovered from
the int8 weight), which halves the weight memory; ``keep_fp16_weight=True``
keeps a [in_features, out_features] fp16 copy for the outlier product instead.
"""
from __future__ import annotations

from typing import Optional

import torch

from .capi import empty_workspace, llmint8_mixed_matmul, llmint8_quantize_weight_colwise, round_up


class Int8Linear(torch.nn.Module):
    """y = x W^T + b with W in int8 (one scale per output feature) and the
    outlier feature dimensions of x (|x| >= threshold in some row) in fp16."""

    def __init__(self, weight: torch.Tensor, bias: Optional[torch.Tensor] = None, threshold: float = 6.0,
                 keep_fp16_weight: bool = False):
        super().__init__()
        if weight.dim() != 2:
            raise ValueError("weight: expected [out_features, in_features]")
        self.out_features, self.in_features = weight.shape
        self.threshold = float(threshold)
        W = weight.detach().to(torch.float16).t().contiguous()  # [K, N], the layout the library quantizes
        K, N = W.shape
        Wq = torch.empty((N, round_up(K, 16)), dtype=torch.int8, device=W.device)
        cs = torch.empty(N, dtype=torch.float32, device=W.device)
        llmint8_quantize_weight_colwise(W, Wq, cs)
        self.register_buffer("weight_int8", Wq)      # [N, round_up(K, 16)], K contiguous
        self.register_buffer("weight_scale", cs)     # [N] fp32 column absmax
        self.register_buffer("weight_fp16", W if keep_fp16_weight else None)
        b = None if bias is None else bias.detach().to(device=W.device, dtype=torch.float16).contiguous()
        self.register_buffer("bias", b)
        self._ws = None
        self._ws_key = None

    @classmethod
    def from_linear(cls, linear: torch.nn.Linear, threshold: float = 6.0,
                    keep_fp16_weight: bool = False) -> "Int8Linear":
        """Convert a (CUDA) nn.Linear at load time."""
        return cls(linear.weight, linear.bias, threshold, keep_fp16_weight)

    def _workspace(self, M: int, device) -> torch.Tensor:
        key = (M, device)
        if self._ws_key != key:
            self._ws = empty_workspace(M, self.out_features, self.in_features, self.in_features, device=device)
            self._ws_key = key
        return self._ws

    def forward(self, x: torch.Tensor) -> torch.Tensor:
        if x.shape[-1] != self.in_features:
            raise ValueError(f"x: expected last dimension {self.in_features}, got {x.shape[-1]}")
        lead = x.shape[:-1]
        x2 = x.reshape(-1, self.in_features)
        if x2.stride(-1) != 1:
            x2 = x2.contiguous()
        M = x2.shape[0]
        y = torch.empty((M, self.out_features), dtype=torch.float16, device=x.device)
        llmint8_mixed_matmul(x2, self.weight_int8, self.weight_scale, self.weight_fp16, self.threshold,
                             self.in_features, y, self._workspace(M, x.device), None, self.bias)
        return y.reshape(*lead, self.out_features)

    def extra_repr(self) -> str:
        return (f"in_features={self.in_features}, out_features={self.out_features}, "
                f"bias={self.bias is not None}, threshold={self.threshold}, "
                f"fp16_weight_kept={self.weight_fp16 is not None}")

    def weight_bytes(self) -> int:
        """Device bytes the layer keeps for its weight (int8 codes, scales,
        the optional fp16 copy)."""
        n = self.weight_int8.numel() + 4 * self.weight_scale.numel()
        if self.weight_fp16 is not None:
            n += 2 * self.weight_fp16.numel()
        return n


__all__ = ["Int8Linear"]
