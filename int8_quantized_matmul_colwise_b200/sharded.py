"""Column-parallel (N-sharded) LLM.int8() matmul over several GPUs.

The pages deploy large models on 8-GPU servers ("Compress your LLMs": OPT-175B
on 8x A100 80 GB in 16-bit, on 8x RTX 3090 24 GB with LLM.int8()).  The split
that needs no exchange before the matmul is by output column: each rank holds
the int8 codes, column scales and fp16 columns of W for its range of output
columns, X is replicated, and since the outlier set O is a function of X alone
(a column of X is an outlier if any of its values reaches the threshold)
every rank finds the same O by itself.  The ranks' Y columns are independent;
one all-gather (NCCL over NVLink) assembles Y.

Column-wise quantization is per column of W, so a rank's codes and scales
are exactly the columns of the full weight's: the sharded result equals the
single-GPU result bit for bit.

One call: each rank's kernels write Y[:, n_r .. n_{r+1}) into slot r of a
gather buffer [world, M, Ns]; ``all_gather_into_tensor`` fills the other
slots; ``llmint8_unshard_columns`` copies the slots into Y [M, N].  Shard
bounds are multiples of 8 columns, so every slot starts 16-byte aligned.

The local step and the reassembly default to this library's CUDA path; the
``local`` / ``unshard`` arguments exist so that the partition and the gather
order can be tested on CPU ranks (gloo) with stand-ins.
"""
from __future__ import annotations

import ctypes
from typing import Callable, List, Optional

from . import capi

ALIGN = 8  # shard bounds are multiples of this many columns (16 bytes of fp16)


def shard_bounds(N: int, world: int, align: int = ALIGN) -> List[int]:
    """Bounds [n_0 = 0, n_1, ..., n_world = N] of the column shards: equal
    shares rounded up to a multiple of ``align`` (the last ranks may get fewer
    columns, or none when N is small)."""
    if N < 1 or world < 1:
        raise ValueError("N and world must be >= 1")
    per = -(-N // world)
    per = -(-per // align) * align
    return [min(N, r * per) for r in range(world + 1)]


def shard_width(N: int, world: int, align: int = ALIGN) -> int:
    """Columns of every slot of the gather buffer (the widest shard)."""
    b = shard_bounds(N, world, align)
    return max(1, max(b[r + 1] - b[r] for r in range(world)))


class ShardedInt8Weight:
    """This rank's share of a weight W [K, N]: output columns [n0, n1),
    converted once at load time to int8 codes (Wq [n1 - n0, ldk]) and column
    scales, plus the fp16 columns W[:, n0:n1] unless ``keep_fp16`` is False
    (then the outlier rows are recovered from the codes)."""

    def __init__(self, W, rank: int, world: int, keep_fp16: bool = True, stream=None,
                 quantize: Optional[Callable] = None):
        if not 0 <= rank < world:
            raise ValueError("rank must be in [0, world)")
        self.K, self.N = W.shape
        self.rank, self.world = rank, world
        self.bounds = shard_bounds(self.N, world)
        self.n0, self.n1 = self.bounds[rank], self.bounds[rank + 1]
        self.width = shard_width(self.N, world)
        if self.n1 > self.n0:
            cols = W[:, self.n0:self.n1].contiguous()
            if quantize is None:
                from . import quantize_weight_colwise
                self.Wq, self.col_scale = quantize_weight_colwise(cols, stream)
            else:
                self.Wq, self.col_scale = quantize(cols)
            self.W = cols if keep_fp16 else None
        else:  # an empty shard (N smaller than world * ALIGN)
            self.Wq = self.col_scale = self.W = None


def gather_buffer(M: int, shard: ShardedInt8Weight, device):
    """The [world, M, Ns] fp16 buffer a call gathers into."""
    import torch
    return torch.empty((shard.world, M, shard.width), dtype=torch.float16, device=device)


def local_into_slot(X, shard: ShardedInt8Weight, buf, tau: float = 6.0, outlier_cap: Optional[int] = None, ws=None,
                    stream=None, local: Optional[Callable] = None):
    """This rank's columns: Y[:, n0:n1] into slot ``shard.rank`` of buf."""
    if shard.n1 <= shard.n0:
        return
    Yr = buf[shard.rank][:, :shard.n1 - shard.n0]
    if local is None:
        from . import mixed_matmul
        mixed_matmul(X, shard.Wq, shard.col_scale, shard.W, tau, outlier_cap, Y=Yr, ws=ws, stream=stream)
    else:
        local(X, shard, tau, Yr)


def sharded_mixed_matmul(X, shard: ShardedInt8Weight, tau: float = 6.0, group=None, outlier_cap: Optional[int] = None,
                         ws=None, stream=None, local: Optional[Callable] = None,
                         unshard: Optional[Callable] = None):
    """Y = X . W over the ranks of ``group``; X [M, K] fp16 replicated on
    every rank; returns Y [M, N] on every rank.  Every rank must call it with
    the same X (the outlier set is then the same everywhere)."""
    import torch
    import torch.distributed as dist
    M, K = X.shape
    buf = gather_buffer(M, shard, X.device)
    local_into_slot(X, shard, buf, tau, outlier_cap, ws, stream, local)
    dist.all_gather_into_tensor(buf.view(-1), buf[shard.rank].reshape(-1), group=group)
    Y = torch.empty((M, shard.N), dtype=torch.float16, device=X.device)
    if unshard is None:
        llmint8_unshard_columns(buf, shard.bounds, Y, stream)
    else:
        unshard(buf, shard.bounds, Y)
    return Y


def llmint8_unshard_columns(blocks, bounds: List[int], Y, stream=None):
    """blocks fp16 [world, M, ld_block] (CUDA) -> Y fp16 [M, N] (CUDA)."""
    import torch
    if blocks.dtype != torch.float16 or Y.dtype != torch.float16 or not blocks.is_cuda or not Y.is_cuda:
        raise TypeError("blocks and Y must be fp16 CUDA tensors")
    if blocks.dim() != 3 or not blocks.is_contiguous() or Y.stride(1) != 1:
        raise ValueError("blocks must be a contiguous [world, M, ld] tensor and Y row-major")
    world, M, ld = blocks.shape
    b = (ctypes.c_int64 * (world + 1))(*bounds)
    capi._check(capi.lib().llmint8_unshard_columns(blocks.data_ptr(), world, M, ld, b, Y.data_ptr(), capi._ld(Y),
                                                  capi._stream(stream)), "llmint8_unshard_columns")
