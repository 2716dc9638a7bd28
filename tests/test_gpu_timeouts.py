"""Failure detection on the GPU without a fault: every wait inside the kernels
is bounded, and a wait that runs out sets the status word's timeout bit and
lets the kernel return, so the context stays usable.

The test hook llmint8_debug_set_waits shortens the bound to 1 ms and makes one
chosen wait wait for an event that never comes (a barrier nothing arrives on,
or one arrival more than the grid has).  Each test checks that the call ends,
that llmint8_check_status reports LLMINT8_ERR_TIMEOUT, and that after the
defaults are restored (and the workspace zero-filled again, since a stalled
grid barrier leaves its counter behind) the next call is bit-exact against
the oracle.
"""
import numpy as np
import pytest

import oracle
import workloads as wl

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

SHORT_NS = 1_000_000  # 1 ms


@pytest.fixture(scope="module")
def L():
    from int8_quantized_matmul_colwise_b200 import _build
    _build.build_library()
    import int8_quantized_matmul_colwise_b200 as lib
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return lib


@pytest.fixture
def stall(L):
    """Set a stall mask with the short bound; always restore the defaults."""
    def set_mask(mask):
        torch.cuda.synchronize()
        L.llmint8_debug_set_waits(SHORT_NS, mask)
    yield set_mask
    torch.cuda.synchronize()
    L.llmint8_debug_set_waits()


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def host(t):
    return t.detach().cpu().numpy()


def y_ok(Y, ref):
    g = host(Y).astype(np.float64)
    r = ref.astype(np.float64)
    assert np.all(np.abs(g - r) <= 1e-3 * np.abs(r) + 1e-3 * np.abs(r).max())


def test_activation_grid_barrier_timeout(L, stall):
    w = wl.get("ragged_129x257x520")
    X = wl.make_x(w)
    Xd = dev(X)
    assert L.llmint8_mixed_matmul_path(Xd, torch.empty((1, 528), dtype=torch.int8, device="cuda"),
                                       w.K)[0] == "act_fused_kernel"
    ws = L.empty_workspace(w.M, 1, w.K, w.K)
    stall(L.capi.STALL_ACT_GRID_BARRIER)
    L.quantize_act_rowwise_outliers(Xd, w.tau, ws=ws)
    st, flags = L.llmint8_check_status(ws)
    assert st == L.capi.ERR_TIMEOUT and flags & L.capi.STATUS_TIMEOUT
    # defaults back, workspace zero-filled: the next call is exact
    L.llmint8_debug_set_waits()
    L.llmint8_workspace_init(ws)
    out = L.quantize_act_rowwise_outliers(Xd, w.tau, ws=ws)
    assert L.llmint8_check_status(ws) == (0, 0)
    O, rs, Xq = oracle.quantize_activation(X, w.tau)
    assert np.array_equal(host(out["Xq"])[:, :w.K], Xq) and np.array_equal(host(out["row_scale"]), rs)
    assert np.array_equal(host(out["outlier_idx"])[:O.size], O)


def test_gemv_decode_weight_wait_timeout(L, stall):
    w = wl.get("decode_m1")
    X, W = wl.make_inputs(w)
    Xd, Wd = dev(X), dev(W)
    Wq, cs = L.quantize_weight_colwise(Wd)
    assert L.llmint8_mixed_matmul_path(Xd, Wq, w.K) == ["decode_gemv_kernel"]
    ws = L.empty_workspace(w.M, w.N, w.K, w.K)
    stall(L.capi.STALL_GEMV_WEIGHT)
    L.mixed_matmul(Xd, Wq, cs, Wd, w.tau, ws=ws)
    st, flags = L.llmint8_check_status(ws)
    assert st == L.capi.ERR_TIMEOUT and flags & L.capi.STATUS_TIMEOUT
    L.llmint8_debug_set_waits()
    Y = L.mixed_matmul(Xd, Wq, cs, Wd, w.tau, ws=ws)
    assert L.llmint8_check_status(ws) == (0, 0)
    y_ok(Y, oracle.mixed_matmul(X, W, w.tau)["Y"])


@pytest.mark.parametrize("name", ["ragged_129x257x520", "ragged_1000x1000x1000"])
def test_gemm_operand_wait_timeout(L, stall, name):
    """The tcgen05 GEMM (CTA pairs for M > 128): the MMA issuer's wait runs
    out, the producer and the epilogue see the abort, copies drain, TMEM is
    freed, the kernel returns."""
    w = wl.get(name)
    X, W = wl.make_inputs(w)
    Xd, Wd = dev(X), dev(W)
    Wq, cs = L.quantize_weight_colwise(Wd)
    assert L.llmint8_mixed_matmul_path(Xd, Wq, w.K)[-1] == "gemm_i8_kernel"
    ws = L.empty_workspace(w.M, w.N, w.K, w.K)
    stall(L.capi.STALL_GEMM_OPERANDS)
    L.mixed_matmul(Xd, Wq, cs, Wd, w.tau, ws=ws)
    st, flags = L.llmint8_check_status(ws)
    assert st == L.capi.ERR_TIMEOUT and flags & L.capi.STATUS_TIMEOUT
    L.llmint8_debug_set_waits()
    Y = L.mixed_matmul(Xd, Wq, cs, Wd, w.tau, ws=ws)
    assert L.llmint8_check_status(ws) == (0, 0)
    y_ok(Y, oracle.mixed_matmul(X, W, w.tau)["Y"])


def test_single_cta_gemm_operand_wait_timeout(L, stall):
    """The single-CTA tile shape (M <= 128)."""
    rng = np.random.default_rng(3)
    X, W, _ = wl.random_small(rng, 100, 1024, 600, 3)
    Xd, Wd = dev(X), dev(W)
    Wq, cs = L.quantize_weight_colwise(Wd)
    ws = L.empty_workspace(100, 600, 1024, 1024)
    stall(L.capi.STALL_GEMM_OPERANDS)
    L.mixed_matmul(Xd, Wq, cs, Wd, 6.0, ws=ws)
    st, _ = L.llmint8_check_status(ws)
    assert st == L.capi.ERR_TIMEOUT
    L.llmint8_debug_set_waits()
    Y = L.mixed_matmul(Xd, Wq, cs, Wd, 6.0, ws=ws)
    assert L.llmint8_check_status(ws) == (0, 0)
    y_ok(Y, oracle.mixed_matmul(X, W, 6.0)["Y"])
