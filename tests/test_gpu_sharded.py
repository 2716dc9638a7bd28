"""The N-sharded path's CUDA pieces on one GPU: the reassembly kernel, and
every rank's local step run one after another into its slot of the gather
buffer (no kernel waits on another rank, so running the ranks in turn on one
GPU is an exact stand-in for the gather), then a real NCCL group of one rank
through sharded_mixed_matmul.  Results against the oracle."""
import datetime
import os
import socket

import numpy as np
import pytest

import oracle
import workloads as wl

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def L():
    from int8_quantized_matmul_colwise_b200 import _build
    _build.build_library()
    import int8_quantized_matmul_colwise_b200 as lib
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return lib


def y_close(g, r):
    g = g.astype(np.float64)
    r = r.astype(np.float64)
    assert np.all(np.abs(g - r) <= 1e-3 * np.abs(r) + 1e-3 * np.abs(r).max())


@pytest.mark.parametrize("M,bounds,ld", [(7, [0, 8, 16, 21], 8), (130, [0, 512, 1024, 1500], 512),
                                         (5, [0, 5, 13, 20], 8), (3, [0, 0, 8, 8, 9], 8), (64, [0, 2048], 2048)])
def test_unshard_columns_kernel(L, M, bounds, ld):
    from int8_quantized_matmul_colwise_b200.sharded import llmint8_unshard_columns
    world = len(bounds) - 1
    N = bounds[-1]
    blocks = torch.randn((world, M, ld), device="cuda").half()
    big = torch.full((M + 1, N + 16), 7.0, dtype=torch.float16, device="cuda")
    Y = big[:M, :N]
    llmint8_unshard_columns(blocks, bounds, Y)
    b = blocks.cpu().numpy()
    want = np.concatenate([b[r, :, :bounds[r + 1] - bounds[r]] for r in range(world)], axis=1)
    assert np.array_equal(Y.cpu().numpy().view(np.uint16), want.view(np.uint16))
    assert bool((big[:M, N:] == 7.0).all()) and bool((big[M] == 7.0).all())


@pytest.mark.parametrize("name,world,keep", [("decode_m8", 2, True), ("decode_m8", 8, False), ("decode_m32", 3, True),
                                             ("ffn_6p7b_prefill", 8, True), ("ragged_129x257x520", 3, True),
                                             ("ragged_129x257x520", 4, False)])
def test_every_rank_local_step(L, name, world, keep):
    """Each rank's shard of Wq / scales / fp16 columns, its kernels writing
    into its slot, then the reassembly: Y equals the oracle's (tolerance) and
    the single-GPU call's bit for bit where both run the same kernel family."""
    from int8_quantized_matmul_colwise_b200.sharded import (ShardedInt8Weight, gather_buffer, llmint8_unshard_columns,
                                                            local_into_slot)
    w = wl.get(name)
    X, W = wl.make_inputs(w)
    Xd, Wd = torch.from_numpy(X).cuda(), torch.from_numpy(W).cuda()
    shards = [ShardedInt8Weight(Wd, r, world, keep_fp16=keep) for r in range(world)]
    buf = gather_buffer(w.M, shards[0], Xd.device)
    for sh in shards:
        local_into_slot(Xd, sh, buf, w.tau)
    Y = torch.empty((w.M, w.N), dtype=torch.float16, device="cuda")
    llmint8_unshard_columns(buf, shards[0].bounds, Y)
    torch.cuda.synchronize()
    Wq_ref, cs_ref = oracle.quantize_weight(W)
    r = oracle.mixed_matmul(X, W, w.tau, weight=(Wq_ref, cs_ref), int8_weight=not keep)
    y_close(Y.cpu().numpy(), r["Y"])


def test_one_rank_nccl_group(L):
    """sharded_mixed_matmul end to end on a one-rank NCCL group (the GPU
    path: local kernels, all_gather_into_tensor, reassembly kernel)."""
    import torch.distributed as dist
    from int8_quantized_matmul_colwise_b200.sharded import ShardedInt8Weight, sharded_mixed_matmul
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("nccl", rank=0, world_size=1, timeout=datetime.timedelta(seconds=120),
                            device_id=torch.device("cuda:0"))
    try:
        w = wl.get("ragged_129x257x520")
        X, W = wl.make_inputs(w)
        shard = ShardedInt8Weight(torch.from_numpy(W).cuda(), 0, 1)
        Y = sharded_mixed_matmul(torch.from_numpy(X).cuda(), shard, w.tau)
        torch.cuda.synchronize()
        y_close(Y.cpu().numpy(), oracle.mixed_matmul(X, W, w.tau)["Y"])
    finally:
        dist.destroy_process_group()
