"""Pins for the CPU oracle: checks against what the pages and mathematics fix.

None of these compares the oracle with itself.  The anchors are: the pages'
worked example (golden file), exact rational arithmetic, numpy's IEEE fp16
conversion, closed forms (error bound of round-to-nearest), the two degenerate
thresholds (tau = inf: pure vector-wise int8; tau = 0: the textbook fp16
matmul), invariants (sign symmetry, power-of-two scaling, column permutation),
the planted structure of the synthetic inputs and brute force in exact
rational arithmetic on tiny shapes.
"""
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------- exact helpers

def rha_exact(x: float, s: float) -> int:
    """round-half-away-from-zero of the exact rational 127*x/s (s > 0)."""
    if s == 0:
        return 0
    xn, xd = float(x).as_integer_ratio()
    sn, sd = float(s).as_integer_ratio()
    num = 127 * xn * sd
    den = xd * sn
    q = (2 * abs(num) + den) // (2 * den)
    return q if num >= 0 else -q


def fp16_all_finite() -> np.ndarray:
    h = np.arange(65536, dtype=np.uint32).astype(np.uint16).view(np.float16)
    return h[np.isfinite(h)]


# ---------------------------------------------------------------- fp16 codec

def test_half_decode_all_patterns_match_numpy():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    got = oracle.half_to_double(bits)
    ref = bits.view(np.float16).astype(np.float64)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])
    # signed zeros keep their sign
    assert np.array_equal(np.signbit(got[~nan]), np.signbit(ref[~nan]))


def test_half_encode_matches_numpy_rne():
    rng = np.random.default_rng(7)
    finite = fp16_all_finite().astype(np.float64)
    finite = np.unique(finite)
    mids = (finite[:-1] + finite[1:]) / 2  # exact midpoints: ties
    near = np.concatenate([mids, np.nextafter(mids, np.inf), np.nextafter(mids, -np.inf)])
    vals = np.concatenate([
        finite, near,
        rng.standard_normal(200000) * 10.0 ** rng.integers(-9, 6, 200000),
        [65504.0, 65519.99, 65520.0, 65536.0, 1e9, -65520.0, 2.0 ** -25, 2.0 ** -26, 3 * 2.0 ** -26,
         np.inf, -np.inf, 0.0, -0.0],
    ])
    got = oracle.double_to_half(vals)
    ref = vals.astype(np.float16)
    assert np.array_equal(got.view(np.uint16), ref.view(np.uint16))


def test_half_encode_ties_go_to_even():
    # 1 + 2^-11 lies halfway between 1 and 1 + 2^-10: even significand is 1.
    assert oracle.double_to_half(np.array([1 + 2.0 ** -11]))[0] == np.float16(1.0)
    # 1 + 3*2^-11 lies halfway between 1+2^-10 (odd) and 1+2^-9 (even).
    assert oracle.double_to_half(np.array([1 + 3 * 2.0 ** -11]))[0] == np.float16(1 + 2.0 ** -9)


# ---------------------------------------------------------------- worked example

def _load_worked_example():
    with open(os.path.join(GOLDEN, "worked_example.txt")) as f:
        rows = [ln.split() for ln in f if ln.strip() and not ln.startswith("#")]
    (value, step, stored, recovered), = rows
    return float(value), float(step), int(stored), float(recovered)


def test_worked_example_from_the_pages():
    value, step, stored, recovered = _load_worked_example()
    # The pages' scale is the quantization step; with the absmax convention the
    # vector absmax is s = 127 * step.  Put s and the value in one fp16 row.
    X = np.array([[127 * step, value]], dtype=np.float16)
    O, rs, Xq = oracle.quantize_activation(X, np.inf)
    assert O.size == 0
    assert rs[0] == np.float32(np.float16(12.7))
    assert Xq[0, 1] == stored
    approx = Xq[0, 1] * float(rs[0]) / 127
    assert round(approx, 2) == recovered
    # the rounding error is the page's point: nonzero, within half a step
    assert 0 < abs(float(X[0, 1]) - approx) <= float(rs[0]) / 254


# ---------------------------------------------------------------- quantizer vs exact arithmetic

SCALES = [65504.0, 127.0, 12.703125, 6.0, 1.984375, 1.0, float(np.float16(0.1)), 2.0 ** -14,
          2.0 ** -24, float(np.float16(3.1e-5)), 1000.5, 0.5]


def _rows_for_scale(s: float, width: int = 2048):
    xs = fp16_all_finite()
    xs = xs[np.abs(xs.astype(np.float64)) <= s]
    per = width - 1
    n_rows = -(-xs.size // per)
    pad = np.zeros(n_rows * per, np.float16)
    pad[:xs.size] = xs
    body = pad.reshape(n_rows, per)
    X = np.concatenate([np.full((n_rows, 1), s, np.float16), body], axis=1)
    return X, xs


@pytest.mark.parametrize("s", SCALES)
def test_quantizer_equals_exact_rational_rounding(s):
    """Every finite fp16 x with |x| <= s quantizes to rha(127x/s) exactly."""
    rng = np.random.default_rng(int(s * 1000) % 2 ** 31)
    X, xs = _rows_for_scale(s)
    O, rs, Xq = oracle.quantize_activation(X, np.inf)
    assert O.size == 0
    assert np.all(rs == np.float32(s))
    got = Xq[:, 1:].ravel()[:xs.size]
    exp = np.array([rha_exact(float(x), s) for x in xs.astype(np.float64)], dtype=np.int64)
    assert np.array_equal(got.astype(np.int64), exp)
    assert got.min() >= -127 and got.max() <= 127
    del rng


def test_random_scales_exact():
    rng = np.random.default_rng(11)
    pos = fp16_all_finite()
    pos = pos[pos > 0]
    for s in rng.choice(pos, 6, replace=False):
        X, xs = _rows_for_scale(float(s))
        _, _, Xq = oracle.quantize_activation(X, np.inf)
        got = Xq[:, 1:].ravel()[:xs.size].astype(np.int64)
        exp = np.array([rha_exact(float(x), float(s)) for x in xs.astype(np.float64)])
        assert np.array_equal(got, exp), float(s)


def test_crafted_ties_round_away_from_zero():
    # s = 127: 127x/s = x exactly, so x = k + 1/2 is a tie -> k + 1 (rha), not RNE.
    k = np.arange(0, 127)
    x = np.concatenate([[127.0], k + 0.5, -(k + 0.5)])
    X = x.astype(np.float16)[None, :]
    _, _, Xq = oracle.quantize_activation(X, np.inf)
    q = Xq[0, 1:].astype(np.int64)
    assert np.array_equal(q[:127], k + 1)
    assert np.array_equal(q[127:], -(k + 1))
    assert q[2] == 3  # 2.5 -> 3 (round-half-even would give 2)
    # s = 63.5: 127x/s = 2x, so x = (k + 1/2)/2 is a tie as well.
    x = np.concatenate([[63.5], (k[:120] + 0.5) / 2])
    _, _, Xq = oracle.quantize_activation(x.astype(np.float16)[None, :], np.inf)
    assert np.array_equal(Xq[0, 1:].astype(np.int64), k[:120] + 1)


# ---------------------------------------------------------------- closed forms and invariants

def _problems():
    rng = np.random.default_rng(5)
    out = [("tiny",) + wl.make_inputs(wl.get("tiny"))]
    for i, (M, K, N, n) in enumerate([(7, 33, 9, 2), (1, 64, 17, 1), (12, 24, 5, 0), (31, 100, 23, 5)]):
        X, W, _ = wl.random_small(rng, M, K, N, n)
        out.append((f"rand{i}", X, W))
    return out


@pytest.mark.parametrize("name,X,W", _problems())
def test_error_bound_half_step(name, X, W):
    """|x - q*s/127| <= s/254 for every non-outlier element (round to nearest)."""
    O, rs, Xq = oracle.quantize_activation(X, 6.0)
    x = X.astype(np.float64)
    s = rs.astype(np.float64)[:, None]
    err = np.abs(127 * x - Xq.astype(np.float64) * s)  # exact in double
    mask = np.ones(X.shape[1], bool)
    mask[O] = False
    assert np.all(err[:, mask] <= s / 2)
    assert np.all(Xq[:, ~mask] == 0)
    Wq, cs = oracle.quantize_weight(W)
    werr = np.abs(127 * W.astype(np.float64) - Wq.astype(np.float64) * cs.astype(np.float64)[None, :])
    assert np.all(werr <= cs.astype(np.float64)[None, :] / 2)


@pytest.mark.parametrize("name,X,W", _problems())
def test_tau_inf_is_pure_vectorwise_int8(name, X, W):
    r = oracle.mixed_matmul(X, W, np.inf)
    assert r["O"].size == 0
    x = X.astype(np.float64)
    w = W.astype(np.float64)
    # row scale = full row absmax; column scale = full column absmax
    assert np.array_equal(r["rs"].astype(np.float64), np.abs(x).max(axis=1))
    assert np.array_equal(r["cs"].astype(np.float64), np.abs(w).max(axis=0))
    # integer product equals numpy's int64 matmul of the same codes
    assert np.array_equal(r["acc"], r["Xq"].astype(np.int64) @ r["Wq"].astype(np.int64))
    # Y approximates X.W within the rigorous quantization error bound
    dx = (r["rs"].astype(np.float64) / 254)[:, None]
    dw = (r["cs"].astype(np.float64) / 254)[None, :]
    bound = np.abs(x).sum(1, keepdims=True) * dw + dx * np.abs(w).sum(0, keepdims=True) + \
        X.shape[1] * dx * dw
    exact = x @ w
    y = r["Y"].astype(np.float64)
    assert np.all(np.abs(r["Yd"] - exact) <= bound * (1 + 1e-9) + 1e-300)
    assert np.all(np.abs(y - exact) <= bound * (1 + 1e-9) + np.abs(r["Yd"]) * 2.0 ** -11 + 2.0 ** -25)


@pytest.mark.parametrize("name,X,W", _problems())
def test_tau_zero_is_the_fp16_matmul(name, X, W):
    r = oracle.mixed_matmul(X, W, 0.0)
    assert np.array_equal(r["O"], np.arange(X.shape[1]))
    assert not r["Xq"].any() and not r["acc"].any()
    exact = X.astype(np.float64) @ W.astype(np.float64)
    assert np.allclose(r["Yd"], exact, rtol=1e-12, atol=1e-12)
    ref16 = exact.astype(np.float16).astype(np.float64)
    y = r["Y"].astype(np.float64)
    assert np.mean(y == ref16) > 0.999
    assert np.all(np.abs(y - ref16) <= np.abs(ref16) * 2.0 ** -10 + 2.0 ** -24)


def test_threshold_is_inclusive():
    X = np.zeros((3, 8), np.float16)
    X[1, 2] = 6.0                     # exactly tau: outlier
    X[2, 5] = np.nextafter(np.float16(6.0), np.float16(0))  # just below: not
    X[0, 7] = -6.0                    # sign does not matter
    assert list(oracle.outlier_columns(X, 6.0)) == [2, 7]


def test_planted_columns_are_detected_on_tiny():
    w = wl.get("tiny")
    X = wl.make_x(w)
    O = oracle.outlier_columns(X, w.tau)
    assert set(wl.planted_columns(w)) <= set(O.tolist())
    assert list(O) == sorted(O)


def test_sign_symmetry_and_power_of_two_scaling():
    X, W = wl.make_inputs(wl.get("tiny"))
    O, rs, Xq = oracle.quantize_activation(X, 6.0)
    On, rsn, Xqn = oracle.quantize_activation(-X, 6.0)
    assert np.array_equal(O, On) and np.array_equal(rs, rsn) and np.array_equal(Xqn, -Xq)
    O2, rs2, Xq2 = oracle.quantize_activation((X.astype(np.float32) * 4).astype(np.float16), 24.0)
    assert np.array_equal(O, O2) and np.array_equal(rs2, rs * 4) and np.array_equal(Xq2, Xq)


def test_column_permutation_invariance():
    rng = np.random.default_rng(3)
    X, W = wl.make_inputs(wl.get("tiny"))
    perm = rng.permutation(X.shape[1])
    a = oracle.mixed_matmul(X, W, 6.0)
    b = oracle.mixed_matmul(X[:, perm], W[perm, :], 6.0)
    assert np.array_equal(np.sort(perm[b["O"]]), a["O"])
    assert np.array_equal(a["rs"], b["rs"])
    assert np.array_equal(a["acc"], b["acc"])
    assert np.allclose(a["Yd"], b["Yd"], rtol=1e-12, atol=1e-13)


def test_zero_and_all_outlier_rows():
    X = np.zeros((3, 16), np.float16)
    X[1, :] = 10.0                       # every column of row 1 is an outlier
    X[2, 3] = 1.0
    O, rs, Xq = oracle.quantize_activation(X, 6.0)
    assert O.size == 16 and not Xq.any()
    assert np.all(rs == 0)
    O, rs, Xq = oracle.quantize_activation(X[[0, 2]], 6.0)
    assert O.size == 0 and rs[0] == 0 and not Xq[0].any() and Xq[1, 3] == 127


def test_accumulator_fits_int32():
    X, W = wl.make_inputs(wl.get("tiny"))
    r = oracle.mixed_matmul(X, W, 6.0)
    assert np.abs(r["acc"]).max() <= 127 * 127 * X.shape[1] < 2 ** 31


def test_gather_matches_fancy_indexing():
    X, W = wl.make_inputs(wl.get("tiny"))
    O = oracle.outlier_columns(X, 6.0)
    Xo, Wo = oracle.gather_outliers(X, O, W)
    assert np.array_equal(Xo.view(np.uint16), X[:, O].view(np.uint16))
    assert np.array_equal(Wo.view(np.uint16), W[O, :].view(np.uint16))


def test_row_subset_equals_full_rows():
    X, W = wl.make_inputs(wl.get("tiny"))
    full = oracle.mixed_matmul(X, W, 6.0)
    rows = np.array([15, 0, 7])
    sub = oracle.mixed_matmul(X, W, 6.0, rows=rows)
    assert np.array_equal(sub["acc"], full["acc"][rows])
    assert np.array_equal(sub["Y"].view(np.uint16), full["Y"][rows].view(np.uint16))


# ---------------------------------------------------------------- brute force, exact arithmetic

def _fp16_round_fraction(v: Fraction) -> float:
    """Nearest fp16 to an exact rational, ties to even (|v| < 65504)."""
    c = np.float16(float(v))
    best = None
    for cand in (np.nextafter(c, np.float16(-np.inf)), c, np.nextafter(c, np.float16(np.inf))):
        d = abs(Fraction(float(cand)) - v)
        key = (d, int(np.array(cand).view(np.uint16)) & 1)
        if best is None or key < best[0]:
            best = (key, float(cand))
    return best[1]


def _brute(X, W, tau):
    x = [[Fraction(float(v)) for v in row] for row in X.astype(np.float64)]
    w = [[Fraction(float(v)) for v in row] for row in W.astype(np.float64)]
    M, K, N = len(x), len(w), len(w[0])
    O = [k for k in range(K) if any(abs(x[i][k]) >= tau for i in range(M))]
    rest = [k for k in range(K) if k not in O]

    def rha(r):
        q = int(abs(r) + Fraction(1, 2))  # floor(|r| + 1/2)
        return q if r >= 0 else -q

    rs = [max([abs(x[i][k]) for k in rest], default=Fraction(0)) for i in range(M)]
    cs = [max(abs(w[k][j]) for k in range(K)) for j in range(N)]
    Xq = [[0 if (k in O or rs[i] == 0) else rha(127 * x[i][k] / rs[i]) for k in range(K)] for i in range(M)]
    Wq = [[0 if cs[j] == 0 else rha(127 * w[k][j] / cs[j]) for j in range(N)] for k in range(K)]
    acc = [[sum(Xq[i][k] * Wq[k][j] for k in range(K)) for j in range(N)] for i in range(M)]
    Y = [[acc[i][j] * rs[i] * cs[j] / 16129 + sum(x[i][k] * w[k][j] for k in O) for j in range(N)]
         for i in range(M)]
    return O, rs, cs, Xq, Wq, acc, Y


@pytest.mark.parametrize("seed", range(6))
def test_brute_force_exact_on_tiny_shapes(seed):
    rng = np.random.default_rng(100 + seed)
    M, K, N = (int(v) for v in rng.integers(1, 7, 3))
    X, W, _ = wl.random_small(rng, M, K, N, int(rng.integers(0, 3)), w_sigma=0.5)
    tau = float(rng.choice([6.0, 1.5, np.inf]))
    O, rs, cs, Xq, Wq, acc, Y = _brute(X, W, tau)
    r = oracle.mixed_matmul(X, W, tau)
    assert r["O"].tolist() == O
    assert [Fraction(float(v)) for v in r["rs"]] == rs
    assert [Fraction(float(v)) for v in r["cs"]] == cs
    assert r["Xq"].tolist() == Xq
    assert r["Wq"].tolist() == Wq
    assert r["acc"].tolist() == acc
    for i in range(M):
        for j in range(N):
            exact = Y[i][j]
            assert abs(Fraction(r["Yd"][i, j]) - exact) <= abs(exact) * Fraction(1, 2 ** 50) + Fraction(1, 2 ** 80)
            assert float(r["Y"][i, j]) == _fp16_round_fraction(exact)


# ---------------------------------------------------------------- generator

def test_chunked_weight_draw_equals_single_draw():
    w = wl.Workload("chk", 4, 37, 29, seed=9)
    a = wl.make_w(w, chunk_rows=5)
    rng = np.random.default_rng(w.seed + 100)
    b = (rng.standard_normal((37, 29), dtype=np.float32) * np.float32(w.w_sigma)).astype(np.float16)
    assert np.array_equal(a.view(np.uint16), b.view(np.uint16))


# ------------------------------------------------------------------ int8-only weights
# The outlier product may use the weight recovered from its int8 form
# (Wq * cs / 127, rounded once to fp16) instead of a kept fp16 copy.

def _ulp16(v: np.ndarray) -> np.ndarray:
    """Spacing of fp16 values at magnitude v (normal or subnormal)."""
    v = np.maximum(np.abs(v.astype(np.float64)), 2.0 ** -14)
    return 2.0 ** (np.floor(np.log2(v)) - 10)


@pytest.mark.parametrize("name,X,W", _problems())
def test_dequantized_weight_within_half_step(name, X, W):
    """|Wd - W| <= cs/254 (the codes' rounding) + half an fp16 ulp at cs (the
    one fp16 rounding); |Wd| <= cs and Wd has the sign of its code."""
    Wq, cs = oracle.quantize_weight(W)
    Wd = oracle.dequantize_weight(Wq, cs).astype(np.float64)
    c = cs.astype(np.float64)[None, :]
    assert np.all(np.abs(Wd - W.astype(np.float64)) <= c / 254 + _ulp16(c) / 2)
    assert np.all(np.abs(Wd) <= c)
    assert np.all(np.sign(Wd) == np.sign(Wq))


def test_dequantized_weight_is_exact_on_code_valued_weights():
    """W = q * 2^-j with a +-127 * 2^-j entry in every column: cs = 127 * 2^-j,
    the codes are q and the recovered weight is W itself, so the int8-only
    outlier product equals the fp16 one bit for bit."""
    rng = np.random.default_rng(41)
    K, N = 96, 40
    q = rng.integers(-127, 128, (K, N))
    q[rng.integers(0, K, N), np.arange(N)] = rng.choice([-127, 127], N)
    for j in (0, 3, 7):
        W = (q * 2.0 ** -j).astype(np.float16)
        Wq, cs = oracle.quantize_weight(W)
        assert np.array_equal(Wq.astype(np.int64), q)
        Wd = oracle.dequantize_weight(Wq, cs)
        assert np.array_equal(Wd.view(np.uint16), W.view(np.uint16))
        X, _, _ = wl.random_small(rng, 9, K, 1, 4)
        a = oracle.mixed_matmul(X, W, 6.0)
        b = oracle.mixed_matmul(X, W, 6.0, int8_weight=True)
        assert a["O"].size > 0
        assert np.array_equal(a["Y"].view(np.uint16), b["Y"].view(np.uint16))


@pytest.mark.parametrize("name,X,W", _problems())
def test_int8_weight_reading_at_tau_limits(name, X, W):
    """tau = +inf: no outlier product, both readings give the same Y; tau = 0:
    Y is the fp16 matmul of X with the recovered weight."""
    a = oracle.mixed_matmul(X, W, np.inf)
    b = oracle.mixed_matmul(X, W, np.inf, int8_weight=True)
    assert np.array_equal(a["Y"].view(np.uint16), b["Y"].view(np.uint16))
    r = oracle.mixed_matmul(X, W, 0.0, int8_weight=True)
    Wd = oracle.dequantize_weight(*oracle.quantize_weight(W)).astype(np.float64)
    assert np.allclose(r["Yd"], X.astype(np.float64) @ Wd, rtol=1e-12, atol=1e-12)


# ------------------------------------------------------------------ linear-layer bias

def test_bias_alone_when_x_is_zero():
    """X = 0: no codes, no outliers, acc = 0, so every row of Y is the bias
    itself (exact in fp16), with the bias indexed by output column."""
    rng = np.random.default_rng(5)
    M, K, N = 7, 40, 23
    W = (rng.standard_normal((K, N)) * 0.02).astype(np.float16)
    b = (rng.standard_normal(N) * 3).astype(np.float16)
    r = oracle.mixed_matmul(np.zeros((M, K), np.float16), W, 6.0, bias=b)
    assert np.array_equal(r["Y"].view(np.uint16), np.broadcast_to(b.view(np.uint16), (M, N)))


@pytest.mark.parametrize("name,X,W", _problems())
def test_bias_on_the_fp16_matmul(name, X, W):
    """tau = 0 (every column an outlier): Y is the fp16 rounding of X W + b,
    X W summed in double."""
    rng = np.random.default_rng(X.shape[0] * 7 + W.shape[1])
    b = (rng.standard_normal(W.shape[1]) * 0.5).astype(np.float16)
    r = oracle.mixed_matmul(X, W, 0.0, bias=b)
    exact = X.astype(np.float64) @ W.astype(np.float64) + b.astype(np.float64)[None, :]
    assert np.allclose(r["Yd"], exact, rtol=1e-12, atol=1e-12)


# ------------------------------------------------------------------ outlier statistics

def test_outlier_stats_on_constructed_placements():
    """Known placements: 7.0 at listed (row, column) pairs, exactly tau once
    (counts: the threshold is inclusive), -inf once, a NaN and a value just
    below tau (neither counts)."""
    X = np.zeros((10, 50), np.float16)
    pairs = [(0, 3), (0, 17), (4, 3), (9, 49), (4, 20), (7, 3)]
    for i, k in pairs:
        X[i, k] = 7.0
    X[2, 30] = -np.inf
    X[5, 5] = np.nan
    X[6, 8] = np.nextafter(np.float16(6.0), np.float16(0))
    X[3, 40] = 6.0
    st = oracle.outlier_stats(X, 6.0)
    assert st == {"values": 8, "columns": 6, "rows": 6}
    assert st["columns"] == oracle.outlier_columns(X, 6.0).size


def test_outlier_stats_at_tau_limits():
    X = wl.make_x(wl.get("tiny"))
    M, K = X.shape
    assert oracle.outlier_stats(X, 0.0) == {"values": M * K, "columns": K, "rows": M}
    assert oracle.outlier_stats(X, np.inf) == {"values": 0, "columns": 0, "rows": 0}


@pytest.mark.parametrize("name,X,W", _problems())
def test_outlier_stats_columns_agree_with_the_outlier_set(name, X, W):
    st = oracle.outlier_stats(X, 6.0)
    O = oracle.outlier_columns(X, 6.0)
    assert st["columns"] == O.size
    assert st["values"] >= st["columns"] and st["values"] >= st["rows"]
    assert st["values"] <= st["rows"] * max(1, O.size)
