"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every function the header declares, sizes workspaces, names statuses, and
rejects invalid arguments before touching the device."""
import ctypes

import pytest

from int8_quantized_matmul_colwise_b200 import _build, capi


@pytest.fixture(scope="module")
def lib():
    _build.build_library()
    return capi.lib()


def test_every_declared_function_is_exported(lib):
    names = capi.header_functions()
    assert len(names) >= 9
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(capi.SIGNATURES), set(names) ^ set(capi.SIGNATURES)


def _c_kind(decl: str):
    """ctypes type a C parameter or return declaration maps to."""
    d = " ".join(decl.replace("const", " ").split())
    if d.startswith("char*") or d.endswith("char*"):
        return ctypes.c_char_p
    if "*" in d:
        return "pointer"
    for c, t in (("int64_t", ctypes.c_int64), ("uint64_t", ctypes.c_uint64), ("uint32_t", ctypes.c_uint32),
                 ("size_t", ctypes.c_size_t), ("float", ctypes.c_float),
                 ("llmint8_status", ctypes.c_int), ("int", ctypes.c_int)):
        if d.split()[0] == c:
            return t
    raise AssertionError(f"unmapped C type: {decl}")


def test_binding_signatures_match_the_header():
    """Every prototype in include/llmint8.h against the binding's ctypes
    signature: same number of parameters, same kind for each, same return."""
    import re
    text = re.sub(r"/\*.*?\*/", "", open(capi.HEADER).read(), flags=re.S)
    text = re.sub(r"#[^\n]*", "", text)
    protos = re.findall(r"([A-Za-z_][\w\s\*]*?)\b(llmint8_[a-z0-9_]+)\s*\(([^)]*)\)\s*;", text)
    assert {n for _, n, _ in protos} == set(capi.SIGNATURES)
    for ret, name, args in protos:
        want_ret, want_args = capi.SIGNATURES[name]
        ret_words = ret.split()
        ret_decl = " ".join(ret_words[-2:]) if ret_words[-1] == "char*" else ret_words[-1]
        assert _c_kind(ret_decl) == want_ret, (name, ret_decl)
        params = [a.strip() for a in args.split(",") if a.strip()]
        assert len(params) == len(want_args), (name, len(params), len(want_args))
        for i, (prm, t) in enumerate(zip(params, want_args)):
            k = _c_kind(prm if "*" in prm else prm.rsplit(" ", 1)[0])
            if k == "pointer":
                assert t is ctypes.c_void_p or issubclass(t, ctypes._Pointer), (name, i, prm)
            else:
                assert k == t, (name, i, prm, t)


def test_status_strings(lib):
    for code, name in capi.STATUS_NAMES.items():
        assert capi.llmint8_status_string(code) == name
    assert capi.llmint8_status_string(99) == "LLMINT8_UNKNOWN_STATUS"


def test_workspace_layout_and_size(lib):
    M, N, K, cap = 2048, 16384, 4096, 4096
    L = capi.llmint8_workspace_layout(M, N, K, cap)
    assert L.ldq == 4096 and L.ldo == 4096
    assert L.total == capi.llmint8_workspace_size(M, N, K, cap)
    regions = sorted([(L.outlier_idx, 4 * cap), (L.row_scale, 4 * M), (L.xq, M * L.ldq), (L.xo, 2 * M * L.ldo)])
    for (a, na), (b, _) in zip(regions, regions[1:]):
        assert a + na <= b
    assert L.xq % 256 == 0 and L.xo % 256 == 0 and L.outlier_idx % 256 == 0
    assert regions[-1][0] + regions[-1][1] <= L.total
    L2 = capi.llmint8_workspace_layout(3, 33, 24, 1)
    assert L2.ldq == 32 and L2.ldo == 8
    # prefill calls (M > 32) end with the tensor-core outlier product's operands,
    # fp16 [M, 256] and [N, 256], past Xo
    assert L.total >= L.xo + 2 * M * L.ldo + 512 * (M + N)
    L3 = capi.llmint8_workspace_layout(33, 1000, 1000, 1000)
    assert L3.total >= L3.xo + 2 * 33 * L3.ldo + 512 * (33 + 1000)


@pytest.mark.parametrize("M,N,K,cap", [(0, 1, 1, 1), (1, 0, 1, 1), (1, 1, 0, 1), (1, 1, 133144, 1),
                                       (1, 1, 8, 9), (1, 1, 8, -1)])
def test_workspace_size_rejects_bad_sizes(lib, M, N, K, cap):
    assert capi.llmint8_workspace_size(M, N, K, cap) == 0


def _mm(lib, **kw):
    a = dict(X=0x1000, M=4, K=32, ldx=32, Wq=0x2000, ldk=32, cs=0x3000, W=0x4000, ldw=16, bias=None, N=16,
             tau=6.0, cap=32, Y=0x5000, ldy=16, ws=0x10000, ws_bytes=1 << 20, stream=None)
    a.update(kw)
    return lib.llmint8_mixed_matmul(a["X"], a["M"], a["K"], a["ldx"], a["Wq"], a["ldk"], a["cs"], a["W"],
                                    a["ldw"], a["bias"], a["N"], a["tau"], a["cap"], a["Y"], a["ldy"], a["ws"],
                                    a["ws_bytes"], a["stream"])


@pytest.mark.parametrize("kw,expect", [
    (dict(X=None), capi.ERR_INVALID_ARG),
    (dict(M=0), capi.ERR_INVALID_ARG),
    (dict(K=133144, ldx=133144, ldk=133152, cap=1), capi.ERR_INVALID_ARG),
    (dict(ldx=31), capi.ERR_INVALID_ARG),
    (dict(ldk=24), capi.ERR_INVALID_ARG),
    (dict(ldk=40), capi.ERR_INVALID_ARG),        # not a multiple of 16
    (dict(Wq=0x2008), capi.ERR_INVALID_ARG),     # not 16-byte aligned
    (dict(ldy=8), capi.ERR_INVALID_ARG),
    (dict(tau=float("nan")), capi.ERR_INVALID_ARG),
    (dict(tau=-1.0), capi.ERR_INVALID_ARG),
    (dict(cap=0), capi.ERR_INVALID_ARG),
    (dict(cap=33), capi.ERR_INVALID_ARG),
    (dict(ws=None), capi.ERR_WORKSPACE),
    (dict(ws=0x10010), capi.ERR_WORKSPACE),      # not 256-byte aligned
    (dict(ws_bytes=1024), capi.ERR_WORKSPACE),
    (dict(bias=0x6001), capi.ERR_INVALID_ARG),   # bias not 2-byte aligned
    (dict(W=None, ldw=0, ws_bytes=1024), capi.ERR_WORKSPACE),  # W = NULL is accepted (int8-only weight)
])
def test_mixed_matmul_rejects_invalid_arguments_on_the_host(lib, kw, expect):
    # these fail validation before any CUDA call, so no device is needed
    assert _mm(lib, **kw) == expect


def test_weight_quant_rejects_invalid_arguments(lib):
    f = lib.llmint8_quantize_weight_colwise
    assert f(None, 4, 4, 4, 0x2000, 16, 0x3000, None) == capi.ERR_INVALID_ARG
    assert f(0x1000, 4, 4, 3, 0x2000, 16, 0x3000, None) == capi.ERR_INVALID_ARG   # ldw < N
    assert f(0x1000, 4, 4, 4, 0x2000, 8, 0x3000, None) == capi.ERR_INVALID_ARG    # ldk % 16
    assert f(0x1000, 20, 4, 4, 0x2000, 16, 0x3000, None) == capi.ERR_INVALID_ARG   # ldk < K


def test_debug_gemm_rejects_invalid_arguments(lib):
    f = lib.llmint8_debug_int8_gemm_i32
    assert f(0x1000, 16, 0x2000, 16, 1, 1, 17, 0x3000, 1, 0x10000, 256, None) == capi.ERR_INVALID_ARG
    assert f(0x1000, 16, 0x2000, 16, 1, 1, 16, 0x3000, 1, 0x10000, 128, None) == capi.ERR_WORKSPACE


def test_debug_path_accumulator_rejects_invalid_arguments(lib):
    f = lib.llmint8_debug_mixed_matmul_i32
    ok = dict(X=0x1000, M=4, K=32, ldx=32, Wq=0x2000, ldk=32, cs=0x3000, N=16, tau=6.0, cap=32, C=0x5000, ldc=16,
              ws=0x10000, ws_bytes=1 << 20)

    def call(**kw):
        a = dict(ok, **kw)
        return f(a["X"], a["M"], a["K"], a["ldx"], a["Wq"], a["ldk"], a["cs"], a["N"], a["tau"], a["cap"], a["C"],
                 a["ldc"], a["ws"], a["ws_bytes"], None)
    assert call(C=None) == capi.ERR_INVALID_ARG
    assert call(ldc=15) == capi.ERR_INVALID_ARG      # ldc < N
    assert call(C=0x5002) == capi.ERR_INVALID_ARG    # C not 4-byte aligned
    assert call(ws_bytes=512) == capi.ERR_WORKSPACE


def test_unshard_rejects_invalid_bounds(lib):
    import ctypes as C
    f = lib.llmint8_unshard_columns

    def call(bounds, world=None, M=4, ld=8, ldy=64):
        b = (C.c_int64 * len(bounds))(*bounds)
        return f(0x1000, len(bounds) - 1 if world is None else world, M, ld, b, 0x2000, ldy, None)
    assert call([1, 8]) == capi.ERR_INVALID_ARG          # bounds[0] != 0
    assert call([0, 8, 4]) == capi.ERR_INVALID_ARG       # decreasing
    assert call([0, 9]) == capi.ERR_INVALID_ARG          # a block wider than ld_block
    assert call([0, 0]) == capi.ERR_INVALID_ARG          # N = 0
    assert call([0, 8, 16], ldy=15) == capi.ERR_INVALID_ARG
    assert call([0, 8], world=0) == capi.ERR_INVALID_ARG
    assert f(None, 1, 4, 8, (C.c_int64 * 2)(0, 8), 0x2000, 8, None) == capi.ERR_INVALID_ARG


def test_debug_set_waits_rejects_a_zero_bound(lib):
    assert lib.llmint8_debug_set_waits(0, 0) == capi.ERR_INVALID_ARG


def test_binding_refuses_host_tensors():
    torch = pytest.importorskip("torch")
    import int8_quantized_matmul_colwise_b200 as L
    W = torch.zeros(8, 8, dtype=torch.float16)
    with pytest.raises(ValueError):
        L.llmint8_quantize_weight_colwise(W, torch.zeros(8, 16, dtype=torch.int8), torch.zeros(8))


def test_kernel_path_query_rejects_invalid_sizes(lib):
    f = lib.llmint8_mixed_matmul_path
    assert f(0, 16, 16, 16, 16, 0x1000) is None        # M < 1
    assert f(4, 16, 16, 8, 16, 0x1000) is None         # ldx < K
    assert f(4, 16, 16, 16, 8, 0x1000) is None         # ldk < K
    assert f(4, 16, 24, 24, 40, 0x1000) is None        # ldk not a multiple of 16
    assert f(4, 16, 16, 16, 16, None) is None          # no X
    assert f(4, 16, 200000, 200000, 200000, 0x1000) is None  # K beyond the int32 accumulator bound


def test_kernel_count_query_rejects_invalid_sizes(lib):
    f = lib.llmint8_mixed_matmul_kernels
    assert f(0, 16, 16, 16, 0x1000) == 0        # M < 1
    assert f(4, 16, 16, 8, 0x1000) == 0         # ldx < K
    assert f(4, 16, 16, 16, None) == 0          # no X
    assert f(4, 16, 200000, 200000, 0x1000) == 0  # K beyond the int32 accumulator bound
