"""Pins for the CPU oracle: what the pages and the mathematics fix.

Each test checks the oracle against something other than itself: values the
pages print (tests/golden, cited there), closed forms, special cases that
reduce to a textbook routine computed independently (numpy), exact rational
arithmetic, the quantisation error bound, and invariants.  No GPU.
"""
from fractions import Fraction

import numpy as np
import pytest

from conftest import read_golden
from int8_mixed_precision_outlier_b200 import synth


def f16(a):
    return np.asarray(a, dtype=np.float32).astype(np.float16)


def ulp16(y):
    """Spacing of fp16 numbers at |y| (subnormal spacing near zero)."""
    y = np.abs(np.asarray(y, dtype=np.float64))
    e = np.floor(np.log2(np.maximum(y, 2.0 ** -14)))
    return 2.0 ** (e - 10)


# ---------------------------------------------------------------- fp16 format

def test_h2f_every_bit_pattern(oracle):
    h = np.arange(65536, dtype=np.uint16)
    got = oracle.h2f(h)
    ref = h.view(np.float16).astype(np.float32)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan].view(np.uint32), ref[~nan].view(np.uint32))


def test_d2h_round_to_nearest_even(oracle):
    rng = np.random.default_rng(1)
    v = np.concatenate([
        rng.standard_normal(20000) * 10.0 ** rng.integers(-9, 5, 20000),
        [0.0, -0.0, 65504.0, 65519.99, 65520.0, -65520.0, 1e6, 2.0 ** -25, 2.0 ** -24,
         3 * 2.0 ** -26, 2.0 ** -14 - 2.0 ** -26],
    ])
    # exact midpoints between neighbouring halves: ties go to the even code
    hs = rng.integers(0, 0x7bff, 5000).astype(np.uint16)
    lo = hs.view(np.float16).astype(np.float64)
    hi = (hs + 1).view(np.float16).astype(np.float64)
    v = np.concatenate([v, (lo + hi) / 2, -(lo + hi) / 2])
    got = oracle.d2h(v).view(np.uint16)
    with np.errstate(over="ignore"):  # the values past 65520 overflow to inf on purpose
        ref = v.astype(np.float16).view(np.uint16)
    assert np.array_equal(got, ref)


# ------------------------------------------------- the pages' printed examples

def test_worked_example_weight_row(oracle):
    g = read_golden("worked_example_quant.txt")
    w = f16([float(s) for s in g["input"]])[None, :]
    Wq, sw = oracle.quantize_weight(w)
    assert Wq[0].tolist() == [int(s) for s in g["codes"]]
    # scale = max_val / 127 in binary32 (max_val is the fp16 value of 8.9)
    assert sw[0] == np.float32(np.float32(w.max()) / np.float32(127.0))


def test_worked_example_activation_row(oracle):
    g = read_golden("worked_example_quant.txt")
    x = f16([float(s) for s in g["input"]])[None, :]
    flag = oracle.detect_outliers(x, float("inf"))
    Xq, sx = oracle.quantize_activations(x, flag)
    assert Xq[0].tolist() == [int(s) for s in g["codes"]]
    # with the page's threshold the 8.9 column becomes an outlier (>= 6) and
    # the row is re-scaled by the largest remaining magnitude (4.7)
    tau = float(read_golden("threshold.txt")["threshold"][0])
    flag6 = oracle.detect_outliers(x, tau)
    assert oracle.compact(flag6).tolist() == [4]
    Xq6, sx6 = oracle.quantize_activations(x, flag6)
    assert Xq6[0, 4] == 0 and Xq6[0, 2] == 127
    assert sx6[0] == np.float32(np.float32(x[0, 2]) / np.float32(127.0))


def test_scale_example(oracle):
    g = read_golden("scale_example.txt")
    amax = float(g["absmax"][0])
    x = f16([[amax, -1.0, 0.5, 0.25]])
    _, sx = oracle.quantize_activations(x, np.zeros(4, np.uint8))
    assert round(float(sx[0]), int(g["decimals"][0])) == float(g["scale_approx"][0])


def test_squash_example_and_its_cure(oracle):
    g = read_golden("squash_example.txt")
    n = int(g["n_normal"][0])
    lo, hi = (float(s) for s in g["normal_range"])
    rng = np.random.default_rng(3)
    row = np.concatenate([rng.uniform(lo, hi, n), [float(g["outlier"][0])]])
    x = f16(row)[None, :]
    # plain symmetric int8 (no outliers removed): normal values squashed to {0, 1}
    Xq, sx = oracle.quantize_activations(x, oracle.detect_outliers(x, float("inf")))
    codes = set(Xq[0, :n].tolist())
    assert codes <= {int(s) for s in g["normal_codes"]}
    assert Xq[0, n] == 127
    # LLM.int8(): the 100.0 column leaves, the rest use their own max
    flag = oracle.detect_outliers(x, float(read_golden("threshold.txt")["threshold"][0]))
    assert oracle.compact(flag).tolist() == [n]
    Xq6, sx6 = oracle.quantize_activations(x, flag)
    assert Xq6[0, n] == 0
    assert np.abs(Xq6[0, :n]).max() == 127
    assert len(set(Xq6[0, :n].tolist())) > 100


# ------------------------------------------------------------ closed forms

def test_threshold_boundary_is_inclusive(oracle):
    below = np.nextafter(np.float16(6.0), np.float16(0.0))
    x = np.array([[6.0, below, -6.0, 0.0, -float(below)]], np.float16)
    assert oracle.compact(oracle.detect_outliers(x, 6.0)).tolist() == [0, 2]


def test_round_half_to_even(oracle):
    # amax 127 gives scale exactly 1, so x/s is x and ties are exact
    x = f16([[127.0, 2.5, 3.5, -2.5, -3.5, 0.5, 1.5, -0.5, 126.5]])
    Xq, sx = oracle.quantize_activations(x, np.zeros(x.shape[1], np.uint8))
    assert sx[0] == 1.0
    assert Xq[0].tolist() == [127, 2, 4, -2, -4, 0, 2, 0, 126]


def test_zero_row_and_all_outlier_row(oracle):
    X = f16([[0, 0, 0, 0], [7.0, 0, 0, 0], [1.0, 2.0, -3.0, 0.5]])
    W = f16([[1, 2, 3, 4], [0.5, -1, 0.25, 2]])
    Wq, sw = oracle.quantize_weight(W)
    Y, im = oracle.matmul(X, Wq, sw, W, 6.0, intermediates=True)
    assert im["idx"].tolist() == [0]
    assert im["sx"][0] == 0.0 and im["sx"][1] == 0.0
    assert not im["Xq"][:2].any()
    # row 1: only the outlier column contributes: 7*W[:,0], exact in fp16
    assert Y[1].tolist() == [7.0, 3.5]
    assert Y[0].tolist() == [0.0, 0.0]


def test_integer_inputs_quantise_exactly(oracle):
    rng = np.random.default_rng(5)
    T, N, K = 7, 9, 32
    # small integers plus one +-127 per row: every scale is exactly 1 and
    # every |Y| stays below the fp16 maximum (127*20*2 + 30*400 < 65504)
    X = rng.integers(-20, 21, (T, K)).astype(np.float64)
    W = rng.integers(-20, 21, (N, K)).astype(np.float64)
    X[:, 0] = 127.0
    W[:, 1] = -127.0
    Xh, Wh = X.astype(np.float16), W.astype(np.float16)
    Wq, sw = oracle.quantize_weight(Wh)
    assert np.all(sw == 1.0) and np.array_equal(Wq, W.astype(np.int8))
    Y, im = oracle.matmul(Xh, Wq, sw, Wh, float("inf"), intermediates=True)
    assert np.all(im["sx"] == 1.0) and np.array_equal(im["Xq"], X.astype(np.int8))
    exact = X.astype(np.int64) @ W.astype(np.int64).T
    assert np.array_equal(Y, exact.astype(np.float64).astype(np.float16))


def test_outlier_free_input_gives_empty_set(oracle):
    rng = np.random.default_rng(7)
    X = f16(np.clip(rng.standard_normal((12, 96)), -5.9, 5.9))
    W = synth.make_weight(20, 96, seed=7)
    Wq, sw = oracle.quantize_weight(W)
    Y, im = oracle.matmul(X, Wq, sw, W, 6.0, intermediates=True)
    assert im["nO"] == 0
    # then Y is plain vector-wise int8: acc * sx * sw with the int product
    # taken independently by numpy
    acc = im["Xq"].astype(np.int64) @ Wq.astype(np.int64).T
    ref = acc.astype(np.float64) * im["sx"].astype(np.float64)[:, None] * \
        sw.astype(np.float64)[None, :]
    assert np.array_equal(Y, ref.astype(np.float16))


def test_tau_inf_is_plain_int8_gemm(oracle):
    X, W = synth.random_case(19, 160, 33, seed=11)
    Wq, sw = oracle.quantize_weight(W)
    Y, im = oracle.matmul(X, Wq, sw, W, float("inf"), intermediates=True)
    assert im["nO"] == 0
    ref = im["Xq"].astype(np.int64) @ Wq.astype(np.int64).T
    assert np.array_equal(im["acc"], ref.astype(np.int32))


def test_tau_zero_is_fp16_gemm(oracle):
    X, W = synth.random_case(13, 96, 40, seed=12)
    Wq, sw = oracle.quantize_weight(W)
    Y, im = oracle.matmul(X, Wq, sw, W, 0.0, intermediates=True)
    assert im["nO"] == 96 and not im["Xq"].any() and not im["acc"].any()
    ref = (X.astype(np.float64) @ W.astype(np.float64).T).astype(np.float16)
    d = np.abs(Y.astype(np.float64) - ref.astype(np.float64))
    assert np.all(d <= ulp16(ref))
    assert np.mean(Y == ref) > 0.995


def test_outlier_part_is_exact(oracle):
    # every fp16 value is an integer multiple of 2^-24, so sums of products are
    # exact rationals; a handful of terms is exact in binary64 too
    X, W = synth.random_case(5, 48, 6, seed=13, n_dims=5, mag=(6.0, 90.0))
    flag = oracle.detect_outliers(X, 6.0)
    idx = oracle.compact(flag)
    assert idx.size >= 5
    yo = oracle.outlier_gemm(X, W, idx)
    for t in range(5):
        for n in range(6):
            s = sum(Fraction(float(X[t, k])) * Fraction(float(W[n, k])) for k in idx)
            assert Fraction(float(yo[t, n])) == s


def test_int32_overflow_is_reported(oracle):
    K = 140000  # 127*127*K > 2^31
    a = np.full((1, K), 127, np.int8)
    with pytest.raises(OverflowError):
        oracle.int8_gemm(a, a)
    assert oracle.int8_gemm(a[:, :133000], a[:, :133000])[0, 0] == 127 * 127 * 133000


# ------------------------------------------------------------- invariants

def test_code_invariants(oracle):
    w = synth.workload("tiny")
    X, W = w["X"], w["W"]
    Wq, sw = oracle.quantize_weight(W)
    Y, im = oracle.matmul(X, Wq, sw, W, 6.0, intermediates=True)
    O = im["idx"]
    assert np.abs(im["Xq"].astype(np.int32)).max() <= 127
    assert not im["Xq"][:, O].any()
    R = np.setdiff1d(np.arange(X.shape[1]), O)
    assert np.all(np.abs(im["Xq"][:, R].astype(np.int32)).max(axis=1) == 127)
    assert np.all(np.abs(Wq.astype(np.int32)).max(axis=1) == 127)
    # outlier columns of Wq meet zero codes of Xq: changing them leaves acc
    Wq2 = Wq.copy()
    Wq2[:, O] = 77
    assert np.array_equal(oracle.int8_gemm(im["Xq"], Wq2), im["acc"])


def test_tiny_config_outlier_set(oracle):
    w = synth.workload("tiny")
    assert oracle.compact(oracle.detect_outliers(w["X"], 6.0)).tolist() == [7, 100]


def test_column_permutation_invariance(oracle):
    X, W = synth.random_case(24, 128, 31, seed=21, n_dims=4)
    Wq, sw = oracle.quantize_weight(W)
    Y, im = oracle.matmul(X, Wq, sw, W, 6.0, intermediates=True)
    p = np.random.default_rng(22).permutation(128)
    Xp, Wp = np.ascontiguousarray(X[:, p]), np.ascontiguousarray(W[:, p])
    Wqp, swp = oracle.quantize_weight(Wp)
    Yp, imp = oracle.matmul(Xp, Wqp, swp, Wp, 6.0, intermediates=True)
    assert sorted(p[imp["idx"]].tolist()) == im["idx"].tolist()
    assert np.array_equal(imp["Xq"], im["Xq"][:, p])
    assert np.array_equal(imp["sx"], im["sx"]) and np.array_equal(swp, sw)
    assert np.array_equal(imp["acc"], im["acc"])
    d = np.abs(Yp.astype(np.float64) - Y.astype(np.float64))
    assert np.all(d <= ulp16(Y))


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_error_bound_against_fp64(oracle, seed):
    """|Y - X W^T| stays within the closed-form quantisation bound.

    With codes q = rint(x/s) and |x/s| <= 127(1 + 2^-24), each regular element
    obeys |x - s q| <= s c, c = 1/2 + 127 * 2^-24 (the binary32 division adds
    at most half an ulp of x/s).  Expanding X W - (X - sx ex)(W - sw ew) gives
      |Y - XW^T| <= sum_{k in R} (|X| sw c + |W| sx c + sx sw c^2)
                    + half an fp16 ulp of the result (+ binary64 slack).
    The scales in the bound are computed here from the definition on the
    inputs, not taken from the oracle.
    """
    T, K, N = 9, 200, 17
    X, W = synth.random_case(T, K, N, seed=30 + seed, n_dims=3, mag=(8.0, 60.0))
    Wq, sw = oracle.quantize_weight(W)
    Y = oracle.matmul(X, Wq, sw, W, 6.0).astype(np.float64)
    Xd, Wd = X.astype(np.float64), W.astype(np.float64)
    exact = Xd @ Wd.T
    R = ~np.any(np.abs(Xd) >= 6.0, axis=0)
    sx_ref = np.abs(Xd[:, R]).max(axis=1) / 127.0
    sw_ref = np.abs(Wd).max(axis=1) / 127.0
    c = 0.5 + 127 * 2.0 ** -24
    bound = (np.abs(Xd[:, R]) @ np.ones((R.sum(), N))) * sw_ref[None, :] * c \
        + sx_ref[:, None] * (np.abs(Wd[:, R]).sum(axis=1))[None, :] * c \
        + R.sum() * sx_ref[:, None] * sw_ref[None, :] * c * c
    bound = bound * (1 + 1e-6) + ulp16(exact) / 2 + 1e-12
    assert np.all(np.abs(Y - exact) <= bound)
    # and the bound is not vacuous: a scale taken over all columns breaks it
    sx_bad = np.abs(Xd).max(axis=1) / 127.0
    Xq_bad = np.clip(np.rint(Xd / sx_bad[:, None]), -127, 127)
    Y_bad = (Xq_bad[:, R] * sx_bad[:, None]) @ (Wq[:, R].astype(np.float64) * sw[:, None]).T \
        + Xd[:, ~R] @ Wd[:, ~R].T
    assert np.any(np.abs(Y_bad - exact) > bound)
