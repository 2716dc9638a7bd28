"""GPU parity: the CUDA path through the C ABI against the CPU oracle.

Bit-exact: Wq, col scales, outlier set and count, row scales, Xq, the gathered
outlier columns and the int32 accumulator.  Y (fp16) within
|Y_gpu - Y_oracle| <= 1e-3 |Y_oracle| + 1e-3 max|Y_oracle|.
Small, ragged, decode, 6.7B FFN and 8192^3 sweep shapes are compared element
by element over the whole matrices; the 175B shape on every intermediate and
on Y of 64 seeded rows plus the first and last row, in the launch
configuration the benchmark times.  (The int32 accumulators of every path and
the quantizer at every kernel that quantizes are in test_gpu_paths.py.)
"""
import numpy as np
import pytest

import oracle
import workloads as wl

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

RTOL = 1e-3
ATOL_REL_MAX = 1e-3


@pytest.fixture(scope="module")
def L():
    from int8_quantized_matmul_colwise_b200 import _build
    _build.build_library()
    import int8_quantized_matmul_colwise_b200 as lib
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return lib


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def host(t):
    return t.detach().cpu().numpy()


def y_close(y_gpu: np.ndarray, y_ref: np.ndarray):
    g = y_gpu.astype(np.float64)
    r = y_ref.astype(np.float64)
    bound = RTOL * np.abs(r) + ATOL_REL_MAX * np.abs(r).max()
    bad = ~(np.abs(g - r) <= bound)
    assert not bad.any(), (f"{bad.sum()} of {bad.size} outside tolerance; worst |d|="
                           f"{np.abs(g - r)[bad].max()} at {np.argwhere(bad)[0]}")


def assert_status_ok(L, ws):
    st, flags = L.llmint8_check_status(ws)
    assert st == 0 and flags == 0, (st, flags)


# ------------------------------------------------------------------ a0: weights

WEIGHT_SHAPES = [(256, 256), (1000, 1000), (4100, 4095), (520, 257), (24, 33), (1, 5), (4096, 4096)]


@pytest.mark.parametrize("K,N", WEIGHT_SHAPES)
def test_weight_quantization_bit_exact(L, K, N):
    rng = np.random.default_rng(K * 7 + N)
    W = (rng.standard_normal((K, N), dtype=np.float32) * 0.02).astype(np.float16)
    W[rng.integers(0, K), :] = 0  # a zero row
    W[:, rng.integers(0, N)] = 0  # a zero column: scale 0, codes 0
    Wq, cs = L.quantize_weight_colwise(dev(W))
    torch.cuda.synchronize()
    Wq_ref, cs_ref = oracle.quantize_weight(W)
    assert np.array_equal(host(cs), cs_ref)
    g = host(Wq)
    assert np.array_equal(g[:, :K], Wq_ref.T)
    assert not g[:, K:].any()


def test_weight_quantization_full_size_ffn(L):
    w = wl.get("ffn_6p7b_prefill")
    W = wl.make_w(w)
    Wq, cs = L.quantize_weight_colwise(dev(W))
    Wq_ref, cs_ref = oracle.quantize_weight(W)
    assert np.array_equal(host(cs), cs_ref)
    assert np.array_equal(host(Wq)[:, :w.K], Wq_ref.T)


# ------------------------------------------------------------------ a1-a4: activations

ACT_WORKLOADS = ["tiny", "decode_m1", "decode_m8", "decode_m32", "ffn_6p7b_prefill", "sweep8k_o1",
                 "ragged_1000x1000x1000", "ragged_2047x4095x4100", "ragged_129x257x520", "ragged_1x1001x1000",
                 "ragged_3x33x24"]


def check_act(L, X, tau, cap=None):
    M, K = X.shape
    out = L.quantize_act_rowwise_outliers(dev(X), tau, cap)
    O, rs, Xq = oracle.quantize_activation(X, tau)
    n = int(host(out["n_outlier"])[0])
    assert n == O.size
    cap_ = K if cap is None else cap
    k = min(n, cap_)
    assert np.array_equal(host(out["outlier_idx"])[:k], O[:k])
    assert np.array_equal(host(out["row_scale"]), rs)
    g = host(out["Xq"])
    assert np.array_equal(g[:, :K], Xq)
    assert not g[:, K:].any()
    Xo_ref, _ = oracle.gather_outliers(X, O[:k])
    assert np.array_equal(host(out["Xo"])[:, :k].view(np.uint16), Xo_ref.view(np.uint16))
    return out


@pytest.mark.parametrize("name", ACT_WORKLOADS)
def test_activation_quantization_bit_exact(L, name):
    w = wl.get(name)
    X = wl.make_x(w)
    out = check_act(L, X, w.tau)
    assert_status_ok(L, out["ws"])
    planted = set(wl.planted_columns(w).tolist())
    if w.M >= 8:
        got = set(host(out["outlier_idx"])[:int(host(out["n_outlier"])[0])].tolist())
        assert planted <= got


@pytest.mark.parametrize("tau", [np.inf, 0.0, 2.5])
def test_activation_thresholds(L, tau):
    X = wl.make_x(wl.get("ragged_129x257x520"))
    check_act(L, X, tau)


SCALES = [65504.0, 127.0, 12.703125, 6.0, 1.984375, 1.0, float(np.float16(0.1)), 2.0 ** -14, 2.0 ** -24, 1000.5]


@pytest.mark.parametrize("s", SCALES)
def test_exact_quantizer_every_fp16_value(L, s):
    """Rows [s, x_1, ...] with every finite fp16 |x| <= s: the division-free
    kernel quantizer equals the oracle's correctly rounded one."""
    h = np.arange(65536, dtype=np.uint32).astype(np.uint16).view(np.float16)
    xs = h[np.isfinite(h) & (np.abs(h.astype(np.float64)) <= s)]
    per = 4095
    rows = -(-xs.size // per)
    body = np.zeros(rows * per, np.float16)
    body[:xs.size] = xs
    X = np.concatenate([np.full((rows, 1), s, np.float16), body.reshape(rows, per)], axis=1)
    check_act(L, X, np.inf)


def test_activation_workspace_reuse_across_shapes(L):
    """One workspace for calls of several row counts (the one-kernel step's
    grid barrier and its two alternating bitmasks) and for a call whose rows
    are not 16-byte aligned (the two-kernel step): every call bit-exact."""
    K, M_max = 512, 300
    ws = L.empty_workspace(M_max, 1, K, K)
    rng = np.random.default_rng(31)
    for M, tau, strided in [(129, 6.0, False), (16, 6.0, False), (300, 3.0, False), (40, 6.0, True),
                            (129, 6.0, False), (1, 0.0, False), (129, np.inf, False)]:
        X, _, _ = wl.random_small(rng, M, K, 1, 3)
        if strided:
            wide = np.zeros((M, K + 1), np.float16)
            wide[:, :K] = X
            Xd = dev(wide)[:, :K]
        else:
            Xd = dev(X)
        out = L.quantize_act_rowwise_outliers(Xd, tau, ws=ws)
        O, rs, Xq = oracle.quantize_activation(X, tau)
        n = int(host(out["n_outlier"])[0])
        assert n == O.size
        assert np.array_equal(host(out["outlier_idx"])[:n], O)
        assert np.array_equal(host(out["row_scale"]), rs)
        assert np.array_equal(host(out["Xq"])[:, :K], Xq)
        Xo_ref, _ = oracle.gather_outliers(X, O)
        assert np.array_equal(host(out["Xo"])[:, :n].view(np.uint16), Xo_ref.view(np.uint16))
    assert_status_ok(L, ws)


@pytest.mark.parametrize("M,K", [(2048, 4096), (300, 512), (1000, 8192)])
def test_activation_outlier_flagged_by_one_row(L, M, K):
    """Column c holds 5.9 (< tau) in every row but one, which holds 7.0: it is
    an outlier column of the call although only one block of rows sees a
    value >= tau in it, and it carries every other row's largest non-outlier
    value until it is excluded.  The one-kernel step quantizes each block of
    rows against the columns that block flagged and must redo the blocks that
    missed column c; the row scales and codes must equal the oracle's."""
    rng = np.random.default_rng(M + K)
    X = rng.standard_normal((M, K)).astype(np.float16)
    c, c2 = 37, K - 3
    X[:, c] = np.float16(5.9)
    X[M // 2, c] = np.float16(7.0)
    X[:, c2] = np.float16(-5.5)
    X[M - 1, c2] = np.float16(-20.0)
    Xd = dev(X)
    if M == 2048:
        assert L.llmint8_mixed_matmul_path(Xd, torch.empty((1, K), dtype=torch.int8, device="cuda"),
                                           K)[0] == "act_fused_kernel"
    out = check_act(L, X, 6.0)
    assert_status_ok(L, out["ws"])
    assert host(out["outlier_idx"])[:int(host(out["n_outlier"])[0])].tolist() == [c, c2]


# (M, K, tau, planted columns): shapes that take the two streaming kernels,
# one per registers-per-thread variant; K = 4104 pads each Xq row by 8 bytes;
# tau = 0.5 flags most columns (more than the 1024 listed in shared memory)
STREAM_CASES = [(3000, 2048, 6.0, 5), (4096, 4096, 6.0, 6), (4096, 4104, 6.0, 9), (2000, 8192, 6.0, 3),
                (600, 12288, 6.0, 25), (200, 16384, 6.0, 7), (3000, 4096, 0.5, 0), (1700, 8192, np.inf, 4)]


@pytest.mark.parametrize("M,K,tau,n_planted", STREAM_CASES)
def test_activation_streaming_kernels(L, M, K, tau, n_planted):
    rng = np.random.default_rng(M * 7 + K)
    X, _, _ = wl.random_small(rng, M, K, 1, n_planted)
    X[M // 3, K // 5] = np.float16(-9.0)  # an outlier column seen by one row only
    Xd = dev(X)
    assert L.llmint8_mixed_matmul_path(Xd, torch.empty((1, L.round_up(K, 16)), dtype=torch.int8, device="cuda"),
                                       K)[:2] == ["scan_stream_kernel", "quantize_stream_kernel"]
    out = check_act(L, X, tau)
    assert_status_ok(L, out["ws"])


@pytest.mark.parametrize("M,K,strided,first", [(2048, 4096, False, "act_fused_kernel"),
                                                (4096, 4096, False, "scan_stream_kernel"),
                                                (300, 4096, True, "scan_columns_kernel"),
                                                (5, 20000, False, "scan_columns_kernel")])
def test_activation_nan_and_inf(L, M, K, strided, first):
    """NaN is never an outlier and codes to 0 (a row of NaN has scale 0);
    +-Inf makes its column an outlier and is gathered as it is: each
    activation kernel against the oracle, Xo compared bit for bit."""
    rng = np.random.default_rng(M + K)
    X = rng.standard_normal((M, K)).astype(np.float16)
    X[1, 3] = np.nan
    X[M - 1, K // 2] = np.nan
    X[2, :] = np.nan
    X[M // 2, 7] = np.inf
    X[0, K - 1] = -np.inf
    if strided:
        wide = np.zeros((M, K + 1), np.float16)
        wide[:, :K] = X
        Xd = dev(wide)[:, :K]
    else:
        Xd = dev(X)
    assert L.llmint8_mixed_matmul_path(Xd, torch.empty((1, L.round_up(K, 16)), dtype=torch.int8, device="cuda"),
                                       K)[0] == first
    out = L.quantize_act_rowwise_outliers(Xd, 6.0)
    O, rs, Xq = oracle.quantize_activation(X, 6.0)
    n = int(host(out["n_outlier"])[0])
    assert n == O.size and {7, K - 1} <= set(O.tolist())
    assert np.array_equal(host(out["outlier_idx"])[:n], O)
    assert np.array_equal(host(out["row_scale"]), rs) and rs[2] == 0
    assert np.array_equal(host(out["Xq"])[:, :K], Xq)
    Xo_ref, _ = oracle.gather_outliers(X, O)
    assert np.array_equal(host(out["Xo"])[:, :n].view(np.uint16), Xo_ref.view(np.uint16))
    assert_status_ok(L, out["ws"])


def test_activation_workspace_reuse_across_paths(L):
    """One workspace through the streaming pair, the one-kernel step and the
    per-row kernels in turn: the call's bitmask must be back to zero after
    every call whichever kernels wrote it."""
    K = 4096
    ws = L.empty_workspace(4096, 1, K, K)
    rng = np.random.default_rng(77)
    seq = [(4096, 6.0, "scan_stream_kernel", False), (40, 6.0, "scan_columns_kernel", True),
           (4096, 0.5, "scan_stream_kernel", False), (129, 6.0, "act_fused_kernel", False),
           (4096, np.inf, "scan_stream_kernel", False), (300, 6.0, "scan_columns_kernel", True),
           (4096, 6.0, "scan_stream_kernel", False)]
    for M, tau, first, strided in seq:
        X, _, _ = wl.random_small(rng, M, K, 1, 4)
        if strided:
            wide = np.zeros((M, K + 1), np.float16)
            wide[:, :K] = X
            Xd = dev(wide)[:, :K]
        else:
            Xd = dev(X)
        assert L.llmint8_mixed_matmul_path(Xd, torch.empty((1, K), dtype=torch.int8, device="cuda"), K)[0] == first
        out = L.quantize_act_rowwise_outliers(Xd, tau, ws=ws)
        O, rs, Xq = oracle.quantize_activation(X, tau)
        n = int(host(out["n_outlier"])[0])
        assert n == O.size
        assert np.array_equal(host(out["outlier_idx"])[:n], O)
        assert np.array_equal(host(out["row_scale"]), rs)
        assert np.array_equal(host(out["Xq"])[:, :K], Xq)
        Xo_ref, _ = oracle.gather_outliers(X, O)
        assert np.array_equal(host(out["Xo"])[:, :n].view(np.uint16), Xo_ref.view(np.uint16))
    assert_status_ok(L, ws)


def test_activation_strided_rows(L):
    X = wl.make_x(wl.get("tiny"))
    wide = np.zeros((X.shape[0], X.shape[1] + 40), np.float16)
    wide[:, 8:8 + X.shape[1]] = X
    t = dev(wide)[:, 8:8 + X.shape[1]]
    out = L.quantize_act_rowwise_outliers(t, 6.0)
    O, rs, Xq = oracle.quantize_activation(X, 6.0)
    assert np.array_equal(host(out["Xq"])[:, :X.shape[1]], Xq)
    assert np.array_equal(host(out["row_scale"]), rs)


# ------------------------------------------------------------------ a5: int8 GEMM (raw accumulator)

GEMM_SHAPES = [(128, 256, 128), (1, 1, 1), (5, 7, 3), (3, 33, 24), (129, 257, 520), (1, 1001, 1000),
               (1000, 1000, 1000), (300, 600, 4096), (2047, 4095, 4100), (256, 512, 8192),
               # decode kernel (M <= 32): split-K over all SMs, uneven K-block split, both padded widths
               (8, 4096, 4096), (16, 4096, 4100), (17, 1000, 1000), (32, 4095, 2048), (33, 520, 256)]


@pytest.mark.parametrize("M,N,K", GEMM_SHAPES)
def test_int8_gemm_accumulator_bit_exact(L, M, N, K):
    rng = np.random.default_rng(M + 3 * N + 7 * K)
    Xq = rng.integers(-127, 128, (M, K), dtype=np.int8)
    Wq = rng.integers(-127, 128, (N, K), dtype=np.int8)
    ldq = L.round_up(K, 16)
    Xp = np.zeros((M, ldq), np.int8)
    Xp[:, :K] = Xq
    Wp = np.zeros((N, ldq), np.int8)
    Wp[:, :K] = Wq
    C = host(L.debug_int8_gemm_i32(dev(Xp), dev(Wp), K))
    rows = None if M * N * K <= 2e9 else wl.sample_rows(M)
    ref = oracle.int8_matmul(Xq, np.ascontiguousarray(Wq.T), rows)
    got = C.astype(np.int64) if rows is None else C[rows].astype(np.int64)
    assert np.array_equal(got, ref)


def test_int8_gemm_extreme_codes(L):
    """All +-127 codes at the largest K of the workloads: the int32 sum
    reaches 127^2 * K without overflow."""
    M, N, K = 130, 260, 12288
    Xq = np.full((M, K), 127, np.int8)
    Xq[1::2] = -127
    Wq = np.full((N, K), 127, np.int8)
    C = host(L.debug_int8_gemm_i32(dev(Xq), dev(Wq), K))
    assert np.all(C[0::2] == 127 * 127 * K) and np.all(C[1::2] == -127 * 127 * K)


K_MAX = 133143  # the largest K the library takes: 127^2 * K < 2^31


def test_int8_gemm_extreme_codes_at_the_largest_k(L):
    """All +-127 codes at K = 133143: the int32 sums reach +-(2^31 - 20201)."""
    M, N, K = 130, 40, K_MAX
    ldq = L.round_up(K, 16)
    Xq = np.zeros((M, ldq), np.int8)
    Xq[:, :K] = 127
    Xq[1::2, :K] = -127
    Wq = np.zeros((N, ldq), np.int8)
    Wq[:, :K] = 127
    C = host(L.debug_int8_gemm_i32(dev(Xq), dev(Wq), K))
    assert 127 * 127 * K < 2 ** 31
    assert np.all(C[0::2] == 127 * 127 * K) and np.all(C[1::2] == -127 * 127 * K)


@pytest.mark.parametrize("M", [2, 130])
def test_mixed_matmul_at_the_largest_k(L, M):
    """The whole path at K = 133143 (long-row activation kernel; split-K
    decode GEMM for M = 2, tcgen05 GEMM for M = 130): X rows of +-0.5 and W
    columns of 2^-10 quantize to +-127 everywhere, so every accumulator is
    +-127^2 K; Y = +-K / 2048, within fp16 range, against the oracle."""
    N, K = 24, K_MAX
    X = np.full((M, K), 0.5, np.float16)
    X[1::2] = -0.5
    W = np.full((K, N), 2.0 ** -10, np.float16)
    Y, ws, v, (Wq, cs), (st, flags) = run_path(L, X, W, np.inf)
    assert st == 0 and flags == 0
    assert np.array_equal(host(v["xq"])[:, :K], np.where(X > 0, 127, -127).astype(np.int8))
    r = oracle.mixed_matmul(X, W, np.inf)
    y_close(host(Y), r["Y"])
    assert np.allclose(host(Y).astype(np.float64)[0], K / 2048.0, rtol=1e-3)


# ------------------------------------------------------------------ a0-a7: the whole path

def run_path(L, X, W, tau, cap=None, rows=None):
    M, K = X.shape
    N = W.shape[1]
    cap = K if cap is None else cap
    Wd = dev(W)
    Wq, cs = L.quantize_weight_colwise(Wd)
    ws = L.empty_workspace(M, N, K, cap)
    Y = L.mixed_matmul(dev(X), Wq, cs, Wd, tau, cap, ws=ws)
    st, flags = L.llmint8_check_status(ws)
    views = L.workspace_views(ws, M, N, K, cap)
    return Y, ws, views, (Wq, cs), (st, flags)


def check_path(L, X, W, tau, rows=None, cap=None):
    M, K = X.shape
    N = W.shape[1]
    Y, ws, v, (Wq, cs), (st, flags) = run_path(L, X, W, tau, cap)
    assert st == 0 and flags == 0, (st, flags)
    Wq_ref, cs_ref = oracle.quantize_weight(W)
    r = oracle.mixed_matmul(X, W, tau, rows=rows, weight=(Wq_ref, cs_ref))
    n = int(host(v["n_outlier"])[0])
    assert n == r["O"].size
    assert np.array_equal(host(v["outlier_idx"])[:n], r["O"])
    assert np.array_equal(host(v["row_scale"]), r["rs"])
    assert np.array_equal(host(v["xq"])[:, :K], r["Xq"])
    assert not host(v["xq"])[:, K:].any()
    if n <= (K if cap is None else cap):  # the gathered outlier columns, bit for bit
        assert np.array_equal(host(v["xo"])[:, :n].view(np.uint16), X[:, r["O"]].view(np.uint16))
    assert np.array_equal(host(cs), cs_ref)
    Wq_g = host(Wq)
    assert np.array_equal(Wq_g[:, :K], Wq_ref.T)
    assert not Wq_g[:, K:].any()
    Yg = host(Y)
    Yg = Yg if rows is None else Yg[rows]
    y_close(Yg, r["Y"])
    return Yg, r


SMALL_PATH = ["tiny", "decode_m1", "decode_m8", "decode_m32", "ragged_1000x1000x1000", "ragged_129x257x520",
              "ragged_1x1001x1000", "ragged_3x33x24", "ragged_2047x4095x4100"]


@pytest.mark.parametrize("name", SMALL_PATH)
def test_mixed_matmul_small_and_ragged(L, name):
    w = wl.get(name)
    X, W = wl.make_inputs(w)
    check_path(L, X, W, w.tau)


@pytest.mark.parametrize("name", ["tiny", "ragged_129x257x520", "ragged_3x33x24"])
def test_mixed_matmul_tau_inf_and_zero(L, name):
    w = wl.get(name)
    X, W = wl.make_inputs(w)
    check_path(L, X, W, np.inf)
    Yg, r = check_path(L, X, W, 0.0)
    assert r["O"].size == w.K  # every column is an outlier: the fp16 matmul


def test_mixed_matmul_accumulator_matches_oracle(L):
    """The int32 accumulator of the whole path equals the oracle's, through
    the raw-accumulator epilogue on the workspace's own Xq and the GPU Wq."""
    w = wl.get("ragged_1000x1000x1000")
    X, W = wl.make_inputs(w)
    Y, ws, v, (Wq, cs), _ = run_path(L, X, W, w.tau)
    C = host(L.debug_int8_gemm_i32(v["xq"], Wq, w.K))
    r = oracle.mixed_matmul(X, W, w.tau)
    assert np.array_equal(C.astype(np.int64), r["acc"])


def test_outlier_overflow_sets_status_and_nan(L):
    w = wl.get("tiny")
    X, W = wl.make_inputs(w)
    Y, ws, v, _, (st, flags) = run_path(L, X, W, w.tau, cap=1)
    assert st == 5 and flags & 1
    assert int(host(v["n_outlier"])[0]) == 2
    assert np.isnan(host(Y).astype(np.float32)).all()
    # the status word is cleared by reading it
    assert L.llmint8_check_status(ws) == (0, 0)


def test_repeat_calls_are_deterministic_and_reuse_workspace(L):
    w = wl.get("ragged_129x257x520")
    X, W = wl.make_inputs(w)
    Wd = dev(W)
    Wq, cs = L.quantize_weight_colwise(Wd)
    ws = L.empty_workspace(w.M, w.N, w.K, w.K)
    Xd = dev(X)
    a = host(L.mixed_matmul(Xd, Wq, cs, Wd, w.tau, ws=ws)).view(np.uint16)
    b = host(L.mixed_matmul(Xd, Wq, cs, Wd, w.tau, ws=ws)).view(np.uint16)
    # a different X through the same workspace, then the first again
    L.mixed_matmul(dev(wl.make_x(wl.get("ragged_129x257x520"))[::-1].copy()), Wq, cs, Wd, 3.0, ws=ws)
    c = host(L.mixed_matmul(Xd, Wq, cs, Wd, w.tau, ws=ws)).view(np.uint16)
    assert np.array_equal(a, b) and np.array_equal(a, c)
    assert_status_ok(L, ws)


def test_decode_repeat_calls_leave_split_k_scratch_at_zero(L):
    """Decode-shaped calls: the one-kernel path of mixed_matmul and the split
    entry points (whose split-K GEMM reduces partial sums in the workspace and
    must leave them at zero) agree bit for bit over repeated calls."""
    w = wl.get("decode_m8")
    X, W = wl.make_inputs(w)
    Wd = dev(W)
    Wq, cs = L.quantize_weight_colwise(Wd)
    ws = L.empty_workspace(w.M, w.N, w.K, w.K)
    Xd = dev(X)
    ys = [host(L.mixed_matmul(Xd, Wq, cs, Wd, w.tau, ws=ws)).view(np.uint16) for _ in range(3)]
    assert np.array_equal(ys[0], ys[1]) and np.array_equal(ys[0], ys[2])
    r = oracle.mixed_matmul(X, W, w.tau)
    y_close(ys[0].view(np.float16), r["Y"])
    # the split entry points on the same data (mixed_gemm with a full-size workspace)
    act = L.quantize_act_rowwise_outliers(Xd, w.tau)
    ws2 = L.empty_workspace(w.M, w.N, w.K, w.K)
    for _ in range(3):
        y2 = host(L.mixed_gemm(act, Wq, cs, Wd, ws=ws2)).view(np.uint16)
        assert np.array_equal(y2, ys[0])
    assert_status_ok(L, ws)
    assert_status_ok(L, ws2)


# (M, N, K) of decode calls: a single CTA; clusters of 8 with empty K slices;
# Xq padding (K % 16 == 8); 16 K blocks per CTA (Wq ring refills); N too wide
# for the one-kernel path (three kernels); a 2-row call at the decode size.
DECODE_SHAPES = [(1, 128, 128), (5, 300, 1032), (17, 520, 2056), (24, 129, 264), (9, 2048, 16384),
                 (32, 1024, 8192), (16, 16384, 4096), (2, 4096, 4096),
                 # matrix-vector kernel (M <= 8, K a multiple of 512 up to 4096, at most 64 Wq rows per CTA;
                 # dp4a products up to 4 rows of X, warp MMAs above): one Wq row per CTA, 61 rows per CTA
                 # (two outputs per thread), one 64-column chunk per warp; the others take the cluster
                 # kernel (too many Wq rows per CTA, K not a multiple of 512, K too large)
                 (1, 100, 512), (4, 9000, 512), (5, 9000, 512), (2, 2000, 1024), (8, 2000, 1024),
                 (3, 4096, 2048), (6, 1500, 4096), (7, 4096, 4096),
                 (8, 16384, 1024), (7, 129, 96), (3, 1000, 16384)]


@pytest.mark.parametrize("M,N,K", DECODE_SHAPES)
def test_decode_shapes(L, M, N, K):
    rng = np.random.default_rng(M * 1000003 + N * 1009 + K)
    X, W, _ = wl.random_small(rng, M, K, N, max(1, K // 700))
    check_path(L, X, W, 6.0)


def test_decode_every_column_an_outlier_and_overflow(L):
    """tau = 0: all 512 columns are outliers, more than the epilogue stages
    (it walks the bitmask for the rest); a cap below n_o gives NaN and the
    overflow bit."""
    rng = np.random.default_rng(77)
    X, W, _ = wl.random_small(rng, 4, 512, 256, 2)
    Yg, r = check_path(L, X, W, 0.0)
    assert r["O"].size == 512
    Y, ws, v, _, (st, flags) = run_path(L, X, W, 6.0, cap=1)
    assert st == 5 and flags & 1
    assert int(host(v["n_outlier"])[0]) == 2
    assert np.isnan(host(Y).astype(np.float32)).all()


def test_decode_unaligned_rows_take_the_three_kernel_path(L):
    """X rows that are not 16-byte aligned (ldx = K + 1) go through the
    scan / quantize / split-K GEMM kernels; same results."""
    M, N, K = 8, 1000, 1000
    rng = np.random.default_rng(5)
    X, W, _ = wl.random_small(rng, M, K, N, 3)
    Xw = np.zeros((M, K + 1), np.float16)
    Xw[:, :K] = X
    Xd = dev(Xw)[:, :K]
    Wd = dev(W)
    Wq, cs = L.quantize_weight_colwise(Wd)
    ws = L.empty_workspace(M, N, K, K)
    Y = host(L.mixed_matmul(Xd, Wq, cs, Wd, 6.0, ws=ws))
    assert_status_ok(L, ws)
    r = oracle.mixed_matmul(X, W, 6.0)
    v = L.workspace_views(ws, M, N, K, K)
    assert np.array_equal(host(v["xq"])[:, :K], r["Xq"])
    y_close(Y, r["Y"])
    Ya = host(L.mixed_matmul(dev(X), Wq, cs, Wd, 6.0))  # the one-kernel path, same bits
    assert np.array_equal(Ya.view(np.uint16), Y.view(np.uint16))


# ------------------------------------------------------------------ full-size workloads

@pytest.mark.parametrize("name", ["ffn_6p7b_prefill", "sweep8k_o0", "sweep8k_o0p1", "sweep8k_o1"])
def test_mixed_matmul_full_size(L, name):
    """The whole Y, Xq, O, rs, Xo, cs and Wq of the 6.7B FFN prefill and of
    the 8192^3 sweeps (tau = 6 and +inf) against the oracle."""
    w = wl.get(name)
    X, W = wl.make_inputs(w)
    check_path(L, X, W, w.tau)
    if name.startswith("sweep"):
        check_path(L, X, W, np.inf)


def test_mixed_matmul_full_size_175b(L):
    """175B hidden shape: every intermediate whole, Y on 64 seeded rows plus
    the first and last (the oracle's int8 matmul over all 4096 rows would be
    4.9e12 multiply-adds)."""
    w = wl.get("hidden_175b")
    X, W = wl.make_inputs(w)
    rows = wl.sample_rows(w.M, n=64)
    check_path(L, X, W, w.tau, rows=rows)


# ------------------------------------------------------------------ int8-only weight (W = NULL)
# No fp16 copy of the weight: the outlier rows are recovered from Wq
# (fp16_RNE(Wq * cs / 127)); the oracle's int8_weight reading.

def check_int8_weight(L, X, W, tau, rows=None, split=False, Xd=None):
    M, K = X.shape
    N = W.shape[1]
    Wq, cs = L.quantize_weight_colwise(dev(W))
    Wq_ref, cs_ref = oracle.quantize_weight(W)
    Xd = dev(X) if Xd is None else Xd
    if split:
        act = L.quantize_act_rowwise_outliers(Xd, tau)
        ws = L.empty_workspace(M, N, K, K)
        Y = host(L.mixed_gemm(act, Wq, cs, None, ws=ws))
    else:
        ws = L.empty_workspace(M, N, K, K)
        Y = host(L.mixed_matmul(Xd, Wq, cs, None, tau, ws=ws))
    assert_status_ok(L, ws)
    r = oracle.mixed_matmul(X, W, tau, rows=rows, weight=(Wq_ref, cs_ref), int8_weight=True)
    y_close(Y if rows is None else Y[rows], r["Y"])
    return Y, r


INT8W_SHAPES = ["tiny", "decode_m1", "decode_m8", "decode_m32", "ragged_1000x1000x1000", "ragged_129x257x520",
                "ragged_1x1001x1000", "ragged_2047x4095x4100", "ragged_3x33x24"]


@pytest.mark.parametrize("name", INT8W_SHAPES)
def test_int8_only_weight_path(L, name):
    w = wl.get(name)
    X, W = wl.make_inputs(w)
    check_int8_weight(L, X, W, w.tau)


@pytest.mark.parametrize("name", ["ragged_129x257x520", "decode_m8", "tiny"])
def test_int8_only_weight_split_entry_points(L, name):
    """mixed_gemm with W = NULL: the prefill GEMM's staged rows (M > 32) and
    the split-K decode GEMM's register rows (M <= 32)."""
    w = wl.get(name)
    X, W = wl.make_inputs(w)
    check_int8_weight(L, X, W, w.tau, split=True)


@pytest.mark.parametrize("M,N,K", [(129, 257, 520), (4, 256, 512), (40, 300, 264)])
def test_int8_only_weight_every_column_an_outlier(L, M, N, K):
    """tau = 0: every column is an outlier, so every recovered row is used
    (several staging passes in the prefill GEMM, the epilogue's reload path in
    the decode kernels)."""
    rng = np.random.default_rng(M + N + K)
    X, W, _ = wl.random_small(rng, M, K, N, 2)
    check_int8_weight(L, X, W, 0.0)


def test_int8_only_weight_three_kernel_decode(L):
    """X rows not 16-byte aligned (the scan / quantize / split-K path)."""
    M, N, K = 8, 1000, 1000
    X, W, _ = wl.random_small(np.random.default_rng(9), M, K, N, 3)
    wide = np.zeros((M, K + 1), np.float16)
    wide[:, :K] = X
    check_int8_weight(L, X, W, 6.0, Xd=dev(wide)[:, :K])


def test_int8_only_weight_full_size_ffn(L):
    w = wl.get("ffn_6p7b_prefill")
    X, W = wl.make_inputs(w)
    check_int8_weight(L, X, W, w.tau, rows=wl.sample_rows(w.M))


# ------------------------------------------------------------------ linear layer: bias fused in the epilogue

def _bias_case(M, N, K, seed):
    rng = np.random.default_rng(seed)
    X, W, _ = wl.random_small(rng, M, K, N, 3)
    b = (rng.standard_normal(N) * 0.5).astype(np.float16)
    return X, W, b


@pytest.mark.parametrize("M,N,K,how", [
    (129, 257, 520, "matmul"),      # prefill GEMM epilogue
    (8, 1000, 1000, "matmul"),      # one-kernel decode (cluster split-K)
    (8, 1024, 2048, "matmul"),      # one-kernel decode (matrix-vector)
    (8, 1000, 1000, "unaligned"),   # three-kernel decode
    (129, 257, 520, "split"),       # mixed_gemm, prefill GEMM
    (8, 1000, 1000, "split"),       # mixed_gemm, split-K decode GEMM
])
def test_bias_every_kernel(L, M, N, K, how):
    X, W, b = _bias_case(M, N, K, M + N + K)
    Wd = dev(W)
    Wq, cs = L.quantize_weight_colwise(Wd)
    bd = dev(b)
    if how == "split":
        act = L.quantize_act_rowwise_outliers(dev(X), 6.0)
        Y = host(L.mixed_gemm(act, Wq, cs, Wd, ws=L.empty_workspace(M, N, K, K), bias=bd))
        assert_status_ok(L, act["ws"])
    else:
        if how == "unaligned":
            wide = np.zeros((M, K + 1), np.float16)
            wide[:, :K] = X
            Xd = dev(wide)[:, :K]
        else:
            Xd = dev(X)
        ws = L.empty_workspace(M, N, K, K)
        Y = host(L.mixed_matmul(Xd, Wq, cs, Wd, 6.0, ws=ws, bias=bd))
        assert_status_ok(L, ws)
    r = oracle.mixed_matmul(X, W, 6.0, bias=b)
    y_close(Y, r["Y"])


@pytest.mark.parametrize("M,N,K,n_out,ldy_pad", [
    (129, 257, 520, 40, 0),      # one round of the chunk-outer epilogue (more than 16 outliers), ragged N
    (300, 512, 1024, 96, 0),     # exactly one full round
    (300, 512, 1024, 97, 8),     # two rounds (partial sums parked in TMEM), TMA stores with a padded ldy
    (100, 600, 2048, 250, 3),    # three rounds, single-CTA tiles, direct stores (rows not 16-byte aligned)
    (200, 300, 8192, 24, 0),     # n_o <= K / 256: the product on the CUDA cores, one round
    (64, 257, 32768, 100, 8),    # on the CUDA cores, two rounds, padded ldy
    (100, 257, 1024, 12, 0),     # 16 or fewer outliers but n_o > K / 256: mma.sync in the one-pass epilogue
    (300, 512, 1024, 260, 0),    # past the tensor-core product's 256 columns: mma.sync rounds on every path
])
def test_many_outliers_epilogue_rounds(L, M, N, K, n_out, ldy_pad):
    """The GEMM epilogue with more than 16 outlier columns: the tile's
    64-column chunks outermost, rounds of up to 96 outlier rows, the bias added
    in the last round, for the fp16 weight and the int8-only weight; the
    16-bit product by mma.sync (n_o > K / 256) and on the CUDA cores.  With
    K / 256 < n_o <= 256 the whole path takes the tensor-core product (tested
    below), so each case also runs the split GEMM entry point with a
    256-byte workspace, which has no room for that product's operands and
    leaves it to the epilogue."""
    rng = np.random.default_rng(M + N + K + n_out)
    X, W, _ = wl.random_small(rng, M, K, N, 0)
    cols = np.sort(rng.choice(K, size=n_out, replace=False))
    X[:, cols] = (rng.standard_normal((M, n_out), dtype=np.float32) * 20.0 + 10.0).astype(np.float16)
    b = (rng.standard_normal(N) * 0.5).astype(np.float16)
    Wd = dev(W)
    Wq, cs = L.quantize_weight_colwise(Wd)
    for keep in (True, False):
        big = torch.zeros((M, N + ldy_pad), dtype=torch.float16, device="cuda")
        Y = big[:, :N]
        ws = L.empty_workspace(M, N, K, K)
        L.mixed_matmul(dev(X), Wq, cs, Wd if keep else None, 6.0, Y=Y, ws=ws, bias=dev(b))
        assert_status_ok(L, ws)
        assert int(L.workspace_views(ws, M, N, K, K)["n_outlier"].item()) >= n_out
        r = oracle.mixed_matmul(X, W, 6.0, bias=b, int8_weight=not keep)
        y_close(host(Y), r["Y"])
        # the epilogue's own product: the split entry point without room for the gathered operands
        act = L.quantize_act_rowwise_outliers(dev(X), 6.0)
        small = torch.zeros(256, dtype=torch.uint8, device="cuda")
        big2 = torch.zeros((M, N + ldy_pad), dtype=torch.float16, device="cuda")
        Y2 = big2[:, :N]
        L.mixed_gemm(act, Wq, cs, Wd if keep else None, Y=Y2, ws=small, bias=dev(b))
        assert_status_ok(L, small)
        y_close(host(Y2), r["Y"])


OM_CASES = [
    (129, 257, 520, 40, 0),      # one block of 64 outlier columns, ragged M and N, one tile per CTA pair
    (257, 520, 4096, 17, 0),     # just past K / 256
    (300, 512, 1024, 64, 0),     # exactly one block
    (300, 512, 1024, 65, 8),     # two blocks, padded ldy
    (300, 512, 1024, 128, 0),    # two full blocks (the most it takes)
    (513, 1000, 1000, 50, 3),    # direct stores (rows not 16-byte aligned), K not a multiple of 128
    (2048, 4096, 1024, 40, 0),   # several tiles per CTA pair: each tile's blocks enter the next tile's main loop
    (1024, 8192, 256, 20, 0),    # short main loops (two blocks): the outlier blocks after the next tile's first
    (4096, 4096, 128, 5, 0),     # one-block main loops: the outlier blocks follow the next tile's whole main loop
    (129, 257, 1024, 12, 0),     # 16 or fewer outliers (one block, mostly zero padding)
    (300, 512, 1024, 200, 0),    # four blocks
    (300, 512, 1024, 256, 0),    # four full blocks (the most it takes)
    (129, 257, 1024, 250, 3),    # four blocks, direct stores
    (100, 600, 2048, 40, 3),     # single-CTA tiles (M <= 128), direct stores
    (64, 1000, 1000, 20, 0),     # single-CTA tiles, ragged N and K
    (128, 4096, 512, 70, 0),     # single-CTA tiles, several tiles per CTA, short main loops
]


@pytest.mark.parametrize("M,N,K,n_out,ldy_pad", OM_CASES)
def test_outlier_product_on_the_tensor_cores(L, M, N, K, n_out, ldy_pad):
    """Prefill GEMMs (CTA pairs and single CTAs) with K / 256 < n_o <= 256:
    the epilogue dequantizes the tile in TMEM and kind::f16 MMAs add the
    outlier product onto it from the gathered Xo and W^T (fp16 weight,
    int8-only weight, the split entry point), with the bias.  Y against the oracle; repeated calls on one workspace give
    the same bits and leave the gather counters at zero."""
    rng = np.random.default_rng(7 * M + N + K + n_out)
    X, W, _ = wl.random_small(rng, M, K, N, 0)
    cols = np.sort(rng.choice(K, size=n_out, replace=False))
    X[:, cols] = (rng.standard_normal((M, n_out), dtype=np.float32) * 20.0 + 10.0).astype(np.float16)
    b = (rng.standard_normal(N) * 0.5).astype(np.float16)
    Wd = dev(W)
    Wq, cs = L.quantize_weight_colwise(Wd)
    ws = L.empty_workspace(M, N, K, K)
    for keep in (True, False):
        r = oracle.mixed_matmul(X, W, 6.0, bias=b, int8_weight=not keep)
        assert r["O"].size == n_out
        first = None
        for rep in range(2):
            big = torch.full((M, N + ldy_pad), float("nan"), dtype=torch.float16, device="cuda")
            Y = big[:, :N]
            L.mixed_matmul(dev(X), Wq, cs, Wd if keep else None, 6.0, Y=Y, ws=ws, bias=dev(b))
            assert_status_ok(L, ws)
            assert not host(ws[16:24]).any()  # the gather counters are back at zero
            y = host(Y)
            y_close(y, r["Y"])
            assert np.isnan(host(big[:, N:]).astype(np.float32)).all()  # nothing past column N
            if first is None:
                first = y
            else:
                assert np.array_equal(y.view(np.uint16), first.view(np.uint16))
    # the split entry points (activation step, then the GEMM on its outputs),
    # both on one workspace, twice: the GEMM's gathered operands must leave the
    # activation step's scratch as the next call needs it
    ref = oracle.mixed_matmul(X, W, 6.0, bias=b)["Y"]
    ws2 = L.empty_workspace(M, N, K, K)
    for rep in range(2):
        act = L.quantize_act_rowwise_outliers(dev(X), 6.0, ws=ws2)
        Y2 = host(L.mixed_gemm(act, Wq, cs, Wd, ws=ws2, bias=dev(b)))
        assert_status_ok(L, ws2)
        assert int(host(act["n_outlier"])[0]) == n_out
        assert not host(ws2[16:24]).any()
        y_close(Y2, ref)


@pytest.mark.parametrize("keep", [False, True])
@pytest.mark.parametrize("lead,K,N", [((2, 3), 520, 300), ((4, 50), 1032, 257), ((1,), 4096, 4096)])
def test_int8_linear_module(L, keep, lead, K, N):
    """Int8Linear.from_linear on a randomly initialised fp16 nn.Linear:
    y = x W^T + b through the C ABI, against the oracle (fp16 or int8-only
    weight reading), for decode- and prefill-shaped inputs with planted
    outlier features."""
    torch.manual_seed(K + N)
    lin = torch.nn.Linear(K, N, bias=True).cuda().half()
    m = L.Int8Linear.from_linear(lin, 6.0, keep_fp16_weight=keep)
    M = int(np.prod(lead))
    rng = np.random.default_rng(M + K)
    X, _, _ = wl.random_small(rng, M, K, 1, max(1, K // 500))
    x = dev(X).reshape(*lead, K)
    y = m(x)
    assert y.shape == (*lead, N) and y.dtype == torch.float16
    W = lin.weight.detach().cpu().numpy().T.copy()
    b = lin.bias.detach().cpu().numpy()
    r = oracle.mixed_matmul(X, W, 6.0, bias=b, int8_weight=not keep)
    y_close(host(y).reshape(M, N), r["Y"])
    fp16_bytes = 2 * K * N
    assert m.weight_bytes() < (fp16_bytes * 0.55 if not keep else fp16_bytes * 1.6)


# ------------------------------------------------------------------ outlier statistics

@pytest.mark.parametrize("name", ["tiny", "decode_m8", "ffn_6p7b_prefill", "ragged_2047x4095x4100", "ragged_3x33x24",
                                  "sweep8k_o1"])
def test_outlier_stats_exact(L, name):
    """The three counts equal the oracle's (integers: exact), for tau 6, 0
    (every value), +inf (none), and twice through one workspace (the scratch
    is returned to zero)."""
    w = wl.get(name)
    X = wl.make_x(w)
    Xd = dev(X)
    ws = L.empty_workspace(1, 1, w.K, w.K)
    for tau in (w.tau, 0.0, np.inf, w.tau):
        assert L.outlier_stats(Xd, tau, ws=ws) == oracle.outlier_stats(X, tau), tau


def test_outlier_stats_strided_rows(L):
    X = wl.make_x(wl.get("ragged_129x257x520"))
    wide = np.zeros((X.shape[0], X.shape[1] + 3), np.float16)
    wide[:, 1:1 + X.shape[1]] = X
    t = dev(wide)[:, 1:1 + X.shape[1]]
    assert L.outlier_stats(t, 6.0) == oracle.outlier_stats(X, 6.0)


def test_kernel_count_query(L):
    """llmint8_mixed_matmul_kernels: 1 on the one-kernel decode path, 2 when
    the activation step is one kernel, 3 otherwise."""
    def count(M, N, K, ldx=None):
        ldx = K if ldx is None else ldx
        X = torch.empty((M, ldx), dtype=torch.float16, device="cuda")[:, :K]
        return L.llmint8_mixed_matmul_kernels(X, N)
    assert count(8, 4096, 4096) == 1
    assert count(2048, 16384, 4096) == 2
    assert count(8192, 8192, 8192) == 3        # X too large for shared memory
    assert count(100, 300, 1000, ldx=1001) == 3  # rows not 16-byte aligned


def test_kernel_path_query(L):
    """llmint8_mixed_matmul_path names the kernels of each path, as many as
    llmint8_mixed_matmul_kernels counts."""
    def path(M, N, K, ldx=None, ldk=None):
        ldx = K if ldx is None else ldx
        ldk = L.round_up(K, 16) if ldk is None else ldk
        X = torch.empty((M, ldx), dtype=torch.float16, device="cuda")[:, :K]
        Wq = torch.empty((N, ldk), dtype=torch.int8, device="cuda")
        p = L.llmint8_mixed_matmul_path(X, Wq, K)
        assert len(p) == L.llmint8_mixed_matmul_kernels(X, N)
        return p
    assert path(1, 4096, 4096) == ["decode_gemv_kernel"]
    assert path(8, 4096, 4096) == ["decode_gemv_kernel"]
    assert path(8, 16384, 1024) == ["decode_fused_kernel"]         # more Wq rows per SM than the kernel holds
    assert path(32, 4096, 4096) == ["decode_fused_kernel"]         # more rows of X
    assert path(2048, 16384, 4096) == ["act_fused_kernel", "gemm_i8_kernel"]
    assert path(8192, 8192, 8192) == ["scan_stream_kernel", "quantize_stream_kernel", "gemm_i8_kernel"]
    assert path(8192, 8192, 8192, ldx=8193) == ["scan_columns_kernel", "quantize_rows_kernel", "gemm_i8_kernel"]
    assert path(4096, 1024, 1024) == ["scan_columns_kernel", "quantize_rows_kernel", "gemm_i8_kernel"]  # K < 2048
    assert path(100, 300, 1000, ldx=1001) == ["scan_columns_kernel", "quantize_rows_kernel", "gemm_i8_kernel"]
    assert path(5, 130, 20000) == ["scan_columns_kernel", "quantize_rows_long_kernel", "gemm_i8_decode_kernel"]


@pytest.mark.parametrize("name", ["ragged_1000x1000x1000", "ffn_6p7b_prefill"])
def test_outlier_overflow_on_the_prefill_path(L, name):
    """A cap below n_o through the one-kernel activation step and the tcgen05
    GEMM: the status bit, the true count and a NaN-filled Y."""
    w = wl.get(name)
    X, W = wl.make_inputs(w)
    n_true = oracle.outlier_columns(X, w.tau).size
    assert n_true >= 2
    Y, ws, v, _, (st, flags) = run_path(L, X, W, w.tau, cap=1)
    assert st == 5 and flags & 1
    assert int(host(v["n_outlier"])[0]) == n_true
    assert np.isnan(host(Y).astype(np.float32)).all()


@pytest.mark.parametrize("M,N,K", [(40, 72, 20000), (5, 130, 20000)])
def test_rows_longer_than_16384(L, M, N, K):
    """K > 16384: the long-row activation kernel (prefill) and the three-kernel
    decode path (the one-kernel plan stops at K = 16384)."""
    rng = np.random.default_rng(K + M)
    X, W, _ = wl.random_small(rng, M, K, N, 20)
    check_path(L, X, W, 6.0)
