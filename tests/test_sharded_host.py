"""The N-sharded (column-parallel) path on CPU ranks: shard bounds, each
rank's share of the weight, the all-gather order and the reassembly, with
world sizes 2 and 3 over gloo.  The local matmul and the reassembly are
stand-ins here (the oracle on the rank's columns; a numpy copy), since the
CUDA kernels need a GPU; the result must equal the single-process oracle bit
for bit, because every output column depends only on X (hence the same
outlier set on every rank) and on its own column of W."""
import os
import socket

import numpy as np
import pytest

import oracle
import workloads as wl
from int8_quantized_matmul_colwise_b200.sharded import (ALIGN, ShardedInt8Weight, shard_bounds, shard_width,
                                                        sharded_mixed_matmul)

torch = pytest.importorskip("torch")


@pytest.mark.parametrize("N,world", [(16384, 8), (4096, 2), (1001, 2), (1001, 3), (20, 3), (10, 3), (1, 4),
                                     (49152, 8), (257, 7)])
def test_shard_bounds_cover_the_columns(N, world):
    b = shard_bounds(N, world)
    assert len(b) == world + 1 and b[0] == 0 and b[-1] == N
    assert all(b[r] <= b[r + 1] for r in range(world))
    assert all(x % ALIGN == 0 or x == N for x in b)  # aligned, or clipped at N
    widths = [b[r + 1] - b[r] for r in range(world)]
    assert max(widths) == shard_width(N, world) or (N < 1 and max(widths) == 0)
    # equal shares up to the alignment: no shard wider than ceil(N / world) rounded up to ALIGN
    assert max(widths) <= -(-(-(-N // world)) // ALIGN) * ALIGN


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _oracle_quantize(cols):
    Wq_kn, cs = oracle.quantize_weight(cols.numpy())
    return torch.from_numpy(np.ascontiguousarray(Wq_kn.T)), torch.from_numpy(cs)


def _oracle_local(X, shard, tau, Yr):
    r = oracle.mixed_matmul(X.numpy(), shard.W.numpy(), tau)
    Yr.copy_(torch.from_numpy(r["Y"]))


def _numpy_unshard(buf, bounds, Y):
    for r in range(len(bounds) - 1):
        Y[:, bounds[r]:bounds[r + 1]] = buf[r, :, :bounds[r + 1] - bounds[r]]


def _rank_main(rank, world, port, M, K, N, out_dir):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        X, W, _ = wl.random_small(np.random.default_rng(M + N + K), M, K, N, 3)
        shard = ShardedInt8Weight(torch.from_numpy(W), rank, world, quantize=_oracle_quantize)
        if shard.n1 > shard.n0:  # this rank's codes and scales are the full weight's columns
            Wq_full, cs_full = oracle.quantize_weight(W)
            assert np.array_equal(shard.Wq.numpy(), Wq_full[:, shard.n0:shard.n1].T)
            assert np.array_equal(shard.col_scale.numpy(), cs_full[shard.n0:shard.n1])
        Y = sharded_mixed_matmul(torch.from_numpy(X), shard, 6.0, local=_oracle_local, unshard=_numpy_unshard)
        np.save(os.path.join(out_dir, f"y{rank}.npy"), Y.numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,M,K,N", [(2, 5, 256, 1001), (3, 4, 128, 20), (3, 3, 64, 10), (2, 33, 520, 4096)])
def test_sharded_matmul_equals_the_single_process_result(tmp_path, world, M, K, N):
    import torch.multiprocessing as mp
    mp.start_processes(_rank_main, args=(world, _free_port(), M, K, N, str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    X, W, _ = wl.random_small(np.random.default_rng(M + N + K), M, K, N, 3)
    ref = oracle.mixed_matmul(X, W, 6.0)["Y"]
    for r in range(world):
        y = np.load(tmp_path / f"y{r}.npy")
        assert np.array_equal(y.view(np.uint16), ref.view(np.uint16)), r
