"""GPU parity of every kernel that runs a configuration, through the C ABI.

* The int32 accumulator of each path, bit for bit against the oracle:
  llmint8_debug_mixed_matmul_i32 runs exactly what llmint8_mixed_matmul runs
  (matrix-vector decode kernel, cluster decode kernel, three-kernel decode
  path, activation step + tcgen05 GEMM) with the epilogue storing the raw sum
  instead of Y.  The int8 product before its outer-product dequantization is
  a separately checkable quantity ("8-bit Matrix Multiplication for Large
  Language Models", Summary & Methodology Analysis).
* The quantizer at every place that quantizes: every finite fp16 value, at
  ten scales including the crafted ties of s = 127 (x = k + 1/2 codes to k + 1,
  rounding half away from zero: "What is 8-bit LLM quantization?", How does
  INT8 quantization work?), through the one-kernel activation step, the row
  kernel (unaligned rows), the long-row kernel (K > 16384), both decode
  kernels and the weight kernel.
* Canaries: guard columns and a guard row around every output a call writes
  must come back untouched, on every path.
"""
import numpy as np
import pytest

import oracle
import workloads as wl

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

SCALES = [65504.0, 127.0, 12.703125, 6.0, 1.984375, 1.0, float(np.float16(0.1)), 2.0 ** -14, 2.0 ** -24, 1000.5]


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


def path_of(L, Xd, Wq, K):
    return L.llmint8_mixed_matmul_path(Xd, Wq, K)


def check_path_acc(L, X, Wq_dev, cs_dev, Wq_ref, tau, Xd=None, expect_path=None, cap=None):
    """Raw int32 accumulator of the path + the workspace intermediates, bit
    for bit against the oracle (Wq_ref in the oracle's [K, N] layout)."""
    M, K = X.shape
    Xd = dev(X) if Xd is None else Xd
    if expect_path is not None:
        assert path_of(L, Xd, Wq_dev, K) == expect_path
    cap = K if cap is None else cap
    C, ws = L.debug_mixed_matmul_i32(Xd, Wq_dev, cs_dev, tau, cap)
    st, flags = L.llmint8_check_status(ws)
    assert st == 0 and flags == 0, (st, flags)
    O, rs, Xq = oracle.quantize_activation(X, tau)
    acc = oracle.int8_matmul(Xq, Wq_ref)
    assert np.array_equal(host(C).astype(np.int64), acc)
    v = L.workspace_views(ws, M, Wq_dev.size(0), K, cap)
    n = int(host(v["n_outlier"])[0])
    assert n == O.size
    assert np.array_equal(host(v["outlier_idx"])[:n], O)
    assert np.array_equal(host(v["row_scale"]), rs)
    assert np.array_equal(host(v["xq"])[:, :K], Xq)
    assert np.array_equal(host(v["xo"])[:, :n].view(np.uint16), X[:, O].view(np.uint16))
    return acc


def weight(L, W):
    Wq, cs = L.quantize_weight_colwise(dev(W))
    Wq_ref, cs_ref = oracle.quantize_weight(W)
    assert np.array_equal(host(Wq)[:, :W.shape[0]], Wq_ref.T) and np.array_equal(host(cs), cs_ref)
    return Wq, cs, Wq_ref


# ------------------------------------------------------------------ path accumulators

@pytest.mark.parametrize("name,expect", [
    ("decode_m1", ["decode_gemv_kernel"]),
    ("decode_m8", ["decode_gemv_kernel"]),
    ("decode_m32", ["decode_fused_kernel"]),
    ("tiny", ["decode_fused_kernel"]),
    ("ragged_129x257x520", ["act_fused_kernel", "gemm_i8_kernel"]),
    ("ragged_1000x1000x1000", None),
    ("ragged_3x33x24", None),
    ("ragged_1x1001x1000", None),
    ("ffn_6p7b_prefill", ["act_fused_kernel", "gemm_i8_kernel"]),
])
def test_path_accumulator_bit_exact(L, name, expect):
    w = wl.get(name)
    X, W = wl.make_inputs(w)
    Wq, cs, Wq_ref = weight(L, W)
    check_path_acc(L, X, Wq, cs, Wq_ref, w.tau, expect_path=expect)


# (M, N, K) shapes of the decode kernels' own parity tests
DECODE_ACC_SHAPES = [(1, 128, 128), (5, 300, 1032), (17, 520, 2056), (24, 129, 264), (9, 2048, 16384),
                     (32, 1024, 8192), (16, 16384, 4096), (2, 4096, 4096), (1, 100, 512), (4, 9000, 512),
                     (5, 9000, 512), (2, 2000, 1024), (8, 2000, 1024), (3, 4096, 2048), (6, 1500, 4096),
                     (7, 4096, 4096), (8, 16384, 1024), (7, 129, 96), (3, 1000, 16384)]


@pytest.mark.parametrize("M,N,K", DECODE_ACC_SHAPES)
def test_decode_path_accumulator_bit_exact(L, M, N, K):
    rng = np.random.default_rng(M * 7919 + N * 31 + K)
    X, W, _ = wl.random_small(rng, M, K, N, max(1, K // 700))
    Wq, cs, Wq_ref = weight(L, W)
    check_path_acc(L, X, Wq, cs, Wq_ref, 6.0)


@pytest.mark.parametrize("M", [1, 2, 4, 5, 8, 16, 32])
def test_decode_extreme_codes(L, M):
    """X = +-1 (every code +-127, rs = 1) and W = +-0.5 (every weight code
    +-127): the decode kernels' int32 sums reach +-127^2 K exactly."""
    K, N = 4096, 4096
    rng = np.random.default_rng(100 + M)
    X = np.where(rng.random((M, K)) < 0.5, -1.0, 1.0).astype(np.float16)
    X[0, :] = 1.0  # row 0: every product +127 * w
    W = np.where(rng.random((K, N)) < 0.5, -0.5, 0.5).astype(np.float16)
    W[:, 0] = 0.5  # column 0 all +127: acc[0, 0] = 127^2 K
    Wq, cs, Wq_ref = weight(L, W)
    acc = check_path_acc(L, X, Wq, cs, Wq_ref, np.inf)
    assert acc[0, 0] == 127 * 127 * K


# ------------------------------------------------------------------ the quantizer at every site

def sweep_values(s):
    """Every finite fp16 x with |x| <= s (both signs)."""
    h = np.arange(65536, dtype=np.uint32).astype(np.uint16).view(np.float16)
    return h[np.isfinite(h) & (np.abs(h.astype(np.float64)) <= s)]


def sweep_rows(s, width, rows_per_call=None):
    """Rows [s, x_1, .., x_{width-1}] holding every value of sweep_values(s);
    returned as a list of row blocks of at most rows_per_call rows."""
    xs = sweep_values(s)
    per = width - 1
    rows = -(-xs.size // per)
    body = np.zeros(rows * per, np.float16)
    body[:xs.size] = xs
    X = np.concatenate([np.full((rows, 1), s, np.float16), body.reshape(rows, per)], axis=1)
    if rows_per_call is None:
        return [X]
    blocks = []
    for i in range(0, rows, rows_per_call):
        b = np.zeros((rows_per_call, width), np.float16)  # all-zero rows pad the last block (rs = 0, codes 0)
        part = X[i:i + rows_per_call]
        b[:part.shape[0]] = part
        blocks.append(b)
    return blocks


def check_act_codes(L, X, Xd, expect_kernel):
    M, K = X.shape
    assert L.llmint8_mixed_matmul_path(Xd, torch.empty((1, L.round_up(K, 16)), dtype=torch.int8,
                                                       device="cuda"), K)[1] == expect_kernel
    out = L.quantize_act_rowwise_outliers(Xd, np.inf)
    O, rs, Xq = oracle.quantize_activation(X, np.inf)
    assert int(host(out["n_outlier"])[0]) == 0
    assert np.array_equal(host(out["row_scale"]), rs)
    assert np.array_equal(host(out["Xq"])[:, :K], Xq)


@pytest.mark.parametrize("s", SCALES)
def test_quantizer_stream_kernel(L, s):
    """quantize_stream_kernel: 4096 rows of 4096 columns (zero rows pad the
    sweep), more than the one-kernel step holds."""
    for X in sweep_rows(s, 4096, rows_per_call=4096):
        check_act_codes(L, X, dev(X), "quantize_stream_kernel")


@pytest.mark.parametrize("s", SCALES)
def test_quantizer_row_kernel_unaligned_rows(L, s):
    """quantize_rows_kernel: X rows not 16-byte aligned (ldx = K + 1)."""
    for X in sweep_rows(s, 4096):
        M, K = X.shape
        wide = np.zeros((M, K + 1), np.float16)
        wide[:, :K] = X
        check_act_codes(L, X, dev(wide)[:, :K], "quantize_rows_kernel")


@pytest.mark.parametrize("s", SCALES)
def test_quantizer_long_row_kernel(L, s):
    """quantize_rows_long_kernel: rows of 20000 columns (K > 16384)."""
    for X in sweep_rows(s, 20000):
        check_act_codes(L, X, dev(X), "quantize_rows_long_kernel")


@pytest.mark.parametrize("s", SCALES)
@pytest.mark.parametrize("rows,N,expect", [(8, 4096, "decode_gemv_kernel"), (3, 1024, "decode_gemv_kernel"),
                                           (16, 1024, "decode_fused_kernel")])
def test_quantizer_in_decode_kernels(L, s, rows, N, expect):
    """The codes each CTA of a one-kernel decode call computes for itself:
    the workspace's Xq (written by the first CTA or cluster) and the int32
    accumulator over random non-zero weight codes (a code off by one in any
    CTA changes that CTA's sums), both bit for bit."""
    rng = np.random.default_rng(int(s * 1000) % 65521 + rows)
    K = 4096
    Wq_ref = rng.integers(1, 128, (K, N), dtype=np.int8) * np.where(rng.random((K, N)) < 0.5, -1, 1).astype(np.int8)
    Wq_dev = torch.zeros((N, K), dtype=torch.int8, device="cuda")
    Wq_dev.copy_(dev(np.ascontiguousarray(Wq_ref.T)))
    cs = torch.ones(N, dtype=torch.float32, device="cuda")
    for X in sweep_rows(s, K, rows):
        check_path_acc(L, X, Wq_dev, cs, Wq_ref, np.inf, expect_path=[expect])


@pytest.mark.parametrize("s", SCALES)
def test_quantizer_weight_kernel(L, s):
    """quantize_weight_colwise_kernel: every value as an entry of W's columns
    [s, x_1, ..]^T (each column's absmax is s)."""
    for X in sweep_rows(s, 4096):
        if X.shape[0] < 2:  # a second, all-zero column (scale 0, codes 0) keeps W two-dimensional in torch
            X = np.vstack([X, np.zeros_like(X)])
        W = np.ascontiguousarray(X.T)  # [4096, columns]
        Wq, cs = L.quantize_weight_colwise(dev(W))
        Wq_ref, cs_ref = oracle.quantize_weight(W)
        assert np.array_equal(host(cs), cs_ref)
        assert np.array_equal(host(Wq)[:, :W.shape[0]], Wq_ref.T)


# ------------------------------------------------------------------ canaries

SENTINEL16 = 0x5A5A


def guarded(shape, dtype, fill, extra_cols):
    """A tensor with `extra_cols` guard columns and one guard row, filled with
    `fill`, and the [rows, cols] view of it a call writes."""
    rows, cols = shape
    big = torch.empty((rows + 1, cols + extra_cols), dtype=dtype, device="cuda")
    big.view(torch.int16 if dtype == torch.float16 else dtype).fill_(fill)
    return big, big[:rows, :cols]


def assert_guards(big, rows, cols, fill):
    b = big.view(torch.int16) if big.dtype == torch.float16 else big
    assert bool((b[:rows, cols:] == fill).all()), "guard columns written"
    assert bool((b[rows, :] == fill).all()), "guard row written"


@pytest.mark.parametrize("M,N,K,path", [
    (1, 4096, 4096, "decode_gemv_kernel"),
    (8, 1000, 1024, "decode_gemv_kernel"),
    (32, 4096, 4096, "decode_fused_kernel"),
    (13, 257, 520, "decode_fused_kernel"),
    (8, 1000, 1000, "three-kernel decode"),
    (129, 257, 520, "gemm_i8_kernel"),
    (100, 4096, 1024, "gemm_i8_kernel"),
    (300, 1000, 1000, "gemm_i8_kernel"),
])
def test_canaries_around_y(L, M, N, K, path):
    """Y written through a strided view (ldy = N + 16, or N + 9 so that rows
    are not 16-byte aligned) with a guard row: no store lands outside [M, N]."""
    rng = np.random.default_rng(M + N + K)
    X, W, _ = wl.random_small(rng, M, K, N, 3)
    Wd = dev(W)
    Wq, cs = L.quantize_weight_colwise(Wd)
    if path == "three-kernel decode":
        wide = np.zeros((M, K + 1), np.float16)
        wide[:, :K] = X
        Xd = dev(wide)[:, :K]
    else:
        Xd = dev(X)
        assert path in L.llmint8_mixed_matmul_path(Xd, Wq, K)
    r = oracle.mixed_matmul(X, W, 6.0)
    for extra in (16, 9):
        big, Y = guarded((M, N), torch.float16, SENTINEL16, extra)
        ws = L.empty_workspace(M, N, K, K)
        L.mixed_matmul(Xd, Wq, cs, Wd, 6.0, Y=Y, ws=ws)
        st, flags = L.llmint8_check_status(ws)
        assert st == 0 and flags == 0
        assert_guards(big, M, N, SENTINEL16)
        g = host(Y).astype(np.float64)
        ref = r["Y"].astype(np.float64)
        assert np.all(np.abs(g - ref) <= 1e-3 * np.abs(ref) + 1e-3 * np.abs(ref).max())


@pytest.mark.parametrize("M,K,strided", [(129, 520, False), (16, 4096, False), (300, 1000, False), (5, 20000, False),
                                         (2048, 4096, False), (300, 1000, True), (7, 4100, True)])
def test_canaries_around_activation_outputs(L, M, K, strided):
    """Xq (guard row; its columns up to the given leading dimension are the
    call's to write), Xo (guard columns past outlier_cap and a guard row), the
    row scales and the outlier list (guard elements) come back untouched, on
    the one-kernel step, the row kernel (unaligned rows) and the long-row
    kernel."""
    rng = np.random.default_rng(M * K)
    X, _, _ = wl.random_small(rng, M, K, 1, 4)
    if strided:
        wide = np.zeros((M, K + 3), np.float16)
        wide[:, 1:K + 1] = X
        Xd = dev(wide)[:, 1:K + 1]
    else:
        Xd = dev(X)
    cap = 8
    ldq = L.round_up(K, 16)
    xq_big, Xq = guarded((M, ldq), torch.int8, 0x5A, 0)
    xo_big, Xo = guarded((M, cap), torch.float16, SENTINEL16, 8)
    rs_big = torch.full((M + 4,), -7.0, dtype=torch.float32, device="cuda")
    o_big = torch.full((cap + 4,), -7, dtype=torch.int32, device="cuda")
    n_o = torch.zeros(1, dtype=torch.int32, device="cuda")
    ws = L.empty_workspace(M, 1, K, cap)
    L.llmint8_quantize_act_rowwise_outliers(Xd, 6.0, Xq, rs_big[:M], o_big[:cap], n_o, Xo, ws)
    st, _ = L.llmint8_check_status(ws)
    assert st == 0
    assert_guards(xq_big, M, ldq, 0x5A)
    assert_guards(xo_big, M, cap, SENTINEL16)
    assert bool((rs_big[M:] == -7.0).all()) and bool((o_big[cap:] == -7).all())
    O, rs, Xq_ref = oracle.quantize_activation(X, 6.0)
    assert int(n_o.item()) == O.size <= cap
    assert np.array_equal(host(Xq)[:, :K], Xq_ref) and np.array_equal(host(rs_big[:M]), rs)
