"""The allocation-free activation entry point against the regular one.

Some callers of this library cannot hand it a device workspace: their device
memory is planned once up front, or they may not call cudaMalloc at call time
(it can synchronise the device).  llmint8_quantize_act_rowwise_outliers_noalloc
keeps its scratch in a fixed device array inside the library instead.  This
file is named so that pytest collects it last; it must pass alone in a fresh
process as well as after the other tests (its first call sets the array up).
"""
import ctypes

import numpy as np
import pytest

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


def _outputs(M, K, cap):
    dev = "cuda"
    return {
        "Xq": torch.full((M, (K + 15) // 16 * 16), 77, dtype=torch.int8, device=dev),
        "row_scale": torch.full((M,), -1.0, dtype=torch.float32, device=dev),
        "outlier_idx": torch.full((cap,), -1, dtype=torch.int32, device=dev),
        "n_outlier": torch.full((1,), -1, dtype=torch.int32, device=dev),
        "Xo": torch.zeros((M, cap), dtype=torch.float16, device=dev),
    }


def _noalloc(L, X, tau, out):
    M, K = X.shape
    stream = torch.cuda.current_stream().cuda_stream
    st = L.capi.lib().llmint8_quantize_act_rowwise_outliers_noalloc(
        X.data_ptr(), M, K, X.stride(0), float(tau), out["Xq"].data_ptr(), out["Xq"].stride(0),
        out["row_scale"].data_ptr(), out["outlier_idx"].data_ptr(), out["outlier_idx"].numel(),
        out["n_outlier"].data_ptr(), out["Xo"].data_ptr(), out["Xo"].stride(0), stream)
    assert st == 0, L.llmint8_status_string(st)


def _same(a, b, n):
    assert torch.equal(a["n_outlier"], b["n_outlier"])
    assert torch.equal(a["outlier_idx"][:n], b["outlier_idx"][:n])
    assert torch.equal(a["row_scale"], b["row_scale"])
    assert torch.equal(a["Xq"], b["Xq"])
    assert torch.equal(a["Xo"][:, :n].view(torch.int16), b["Xo"][:, :n].view(torch.int16))


@pytest.mark.parametrize("names", [("ffn_6p7b_prefill", "ragged_129x257x520"), ("decode_m8", "tiny")])
def test_noalloc_matches_workspace_entry_on_two_calls(L, names):
    for name in names:  # two calls in a row through the same device array
        w = wl.get(name)
        X = torch.from_numpy(wl.make_x(w)).cuda()
        cap = w.K
        ref = L.quantize_act_rowwise_outliers(X, w.tau, cap)
        got = _outputs(w.M, w.K, cap)
        _noalloc(L, X, w.tau, got)
        torch.cuda.synchronize()
        n = int(ref["n_outlier"].item())
        ref_out = {k: ref[k] for k in ("Xq", "row_scale", "outlier_idx", "n_outlier", "Xo")}
        _same(got, ref_out, n)


@pytest.mark.parametrize("M,K", [(3, 20000), (2, 61440)])
def test_noalloc_long_rows_and_the_largest_k(L, M, K):
    """Rows longer than 16384 columns (the long-row kernel) and K at the
    array's limit, where the per-block counters and the outlier bitmask sit
    at the end of the array; a few planted outlier columns; two calls."""
    rng = np.random.default_rng(K + M)
    for call in range(2):
        X = (rng.standard_normal((M, K), dtype=np.float32)).astype(np.float16)
        cols = np.sort(rng.choice(K, size=5, replace=False))
        cols[-1] = K - 1  # the last column, in the last bitmask word
        X[:, cols] = (X[:, cols].astype(np.float32) * 20.0).astype(np.float16)
        X[0, cols] = 7.5  # with two rows a x20 column can stay below the threshold; make each one an outlier
        Xd = torch.from_numpy(X).cuda()
        ref = L.quantize_act_rowwise_outliers(Xd, 6.0, K)
        got = _outputs(M, K, K)
        _noalloc(L, Xd, 6.0, got)
        torch.cuda.synchronize()
        n = int(ref["n_outlier"].item())
        assert set(cols.tolist()) <= set(ref["outlier_idx"][:n].tolist())
        _same(got, {k: ref[k] for k in ("Xq", "row_scale", "outlier_idx", "n_outlier", "Xo")}, n)


def test_noalloc_allocates_nothing_at_call_time(L):
    """After one warm-up call, further calls leave both torch's allocator and
    the device's free memory unchanged."""
    w = wl.get("ragged_129x257x520")
    X = torch.from_numpy(wl.make_x(w)).cuda()
    out = _outputs(w.M, w.K, w.K)
    _noalloc(L, X, w.tau, out)
    torch.cuda.synchronize()
    before_torch = torch.cuda.memory_allocated()
    before_free = torch.cuda.mem_get_info()[0]
    for _ in range(5):
        _noalloc(L, X, w.tau, out)
    torch.cuda.synchronize()
    assert torch.cuda.memory_allocated() == before_torch
    assert torch.cuda.mem_get_info()[0] == before_free


def test_noalloc_rejects_k_beyond_its_array(L):
    M, K = 2, 61441
    X = torch.zeros((M, K), dtype=torch.float16, device="cuda")
    out = _outputs(M, K, 1)
    st = L.capi.lib().llmint8_quantize_act_rowwise_outliers_noalloc(
        X.data_ptr(), M, K, K, 6.0, out["Xq"].data_ptr(), out["Xq"].stride(0), out["row_scale"].data_ptr(),
        out["outlier_idx"].data_ptr(), 1, out["n_outlier"].data_ptr(), out["Xo"].data_ptr(), 1,
        torch.cuda.current_stream().cuda_stream)
    assert st == 3  # LLMINT8_ERR_WORKSPACE
    assert int(out["n_outlier"].item()) == -1  # nothing ran
