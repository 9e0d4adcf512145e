"""Pins of the CPU oracle for the variants built on the LLM.int8() path
(SmoothQuant W8A8, FP8 E4M3 decomposition, stored outlier-weight columns):
closed forms, the exact equivalence the transform rests on, special cases that
reduce to the pinned LLM.int8() oracle or to a library routine, and
quantisation error bounds against fp64 brute force.  No GPU.
"""
from fractions import Fraction

import numpy as np
import pytest

from int8_mixed_precision_outlier_b200 import synth


@pytest.fixture(scope="module")
def nx():
    from oracle import oracle_next as O
    O.build()
    return O


def ulp16(y):
    y = np.abs(np.asarray(y, dtype=np.float64))
    return 2.0 ** (np.floor(np.log2(np.maximum(y, 2.0 ** -14))) - 10)


def f32(x):
    return np.float32(x)


# =================================================================== SmoothQuant

def test_column_absmax(nx):
    X, _ = synth.make_activations(37, 96, seed=1, n_dims=3)
    assert np.array_equal(nx.column_absmax(X), np.abs(X.astype(np.float32)).max(axis=0))


def test_smooth_factor_closed_forms(nx):
    ax = np.array([4.0, 100.0, 0.0, 9.0, 1.0], np.float32)
    aw = np.array([0.25, 0.01, 0.5, 0.0, 1.0], np.float32)
    s = nx.smooth_factors(ax, aw, 0.5)
    # sqrt(4)/sqrt(0.25) = 4; sqrt(100)/sqrt(0.01) = 100; zero channels keep 1
    assert s.tolist() == [4.0, 100.0, 1.0, 1.0, 1.0]
    # alpha = 1: s = max|X_j| (all difficulty to the weights); alpha = 0: s = 1 / max|W_j|
    assert nx.smooth_factors(ax, aw, 1.0).tolist() == [4.0, 100.0, 1.0, 1.0, 1.0]
    s0 = nx.smooth_factors(ax, aw, 0.0)
    assert s0[0] == f32(1.0) / f32(0.25) and s0[1] == f32(1.0) / f32(0.01)
    # a general alpha is powf on both sides
    s3 = nx.smooth_factors(np.array([8.0], np.float32), np.array([2.0], np.float32), 0.25)
    assert abs(float(s3[0]) - 8.0 ** 0.25 / 2.0 ** 0.75) <= 4e-7


def smoothed(X, W, s):
    """X diag(s)^-1 and diag(s) W in binary32, as the oracle forms them."""
    Xs = X.astype(np.float32) / s[None, :]
    Ws = W.astype(np.float32) * s[None, :]
    return Xs, Ws


def test_alpha_half_balances_both_sides(nx):
    """[P2] Q10: at alpha = 0.5 the factor splits the range evenly: after the
    transform every channel's activation maximum equals its weight maximum
    (ax / s = sqrt(ax aw) = aw s), up to the roundings of s and the products."""
    X, _ = synth.make_activations(64, 256, seed=2, n_dims=6, mag=(20.0, 90.0))
    W = synth.make_weight(96, 256, seed=2, sigma=0.03)
    s = nx.smooth_factors(nx.column_absmax(X), nx.column_absmax(W), 0.5)
    Xs, Ws = smoothed(X, W, s)
    mx, mw = np.abs(Xs).max(axis=0), np.abs(Ws).max(axis=0)
    assert np.all(np.abs(mx - mw) <= 4 * 2.0 ** -23 * mw)
    # the outlier channels are the ones pulled down most
    big = np.argsort(-nx.column_absmax(X))[:6]
    assert np.all(s[big] > np.median(s) * 3)


def test_transform_is_exact_before_quantisation(nx):
    """[P2] Q9: (X diag(s)^-1)(diag(s) W)^T = X W^T; with binary32 roundings
    of the scaled operands the product moves by at most 2^-23 relative per term."""
    X, _ = synth.make_activations(16, 128, seed=3, n_dims=4)
    W = synth.make_weight(40, 128, seed=3)
    s = nx.smooth_factors(nx.column_absmax(X), nx.column_absmax(W), 0.5)
    Xs, Ws = smoothed(X, W, s)
    exact = X.astype(np.float64) @ W.astype(np.float64).T
    moved = Xs.astype(np.float64) @ Ws.astype(np.float64).T
    bound = 2.0 ** -23 * (np.abs(X.astype(np.float64)) @ np.abs(W.astype(np.float64)).T) * 1.01
    assert np.all(np.abs(moved - exact) <= bound)


def test_unit_factors_reduce_to_vector_wise_int8(nx, oracle):
    """With s = 1 the W8A8 matmul is the LLM.int8() matmul with no outlier
    columns (threshold inf): same codes, scales and Y bit for bit."""
    X, W = synth.random_case(12, 160, 33, seed=4)
    ones = np.ones(160, np.float32)
    Wq, sw = nx.smooth_quantize_weight(W, ones)
    Wq_b, sw_b = oracle.quantize_weight(W)
    assert np.array_equal(Wq, Wq_b) and np.array_equal(sw.view(np.uint32), sw_b.view(np.uint32))
    Y, im = nx.smoothquant_matmul(X, ones, Wq, sw, intermediates=True)
    Y_b, im_b = oracle.matmul(X, Wq_b, sw_b, W, float("inf"), intermediates=True)
    assert np.array_equal(im["Xq"], im_b["Xq"]) and np.array_equal(im["acc"], im_b["acc"])
    assert np.array_equal(Y.view(np.uint16), Y_b.view(np.uint16))


def test_power_of_two_factors_commute_with_quantisation(nx, oracle):
    """Factors that are powers of two scale exactly: the codes of X diag(s)^-1
    and of diag(s) W equal the oracle's codes of the pre-scaled fp16 matrices."""
    rng = np.random.default_rng(5)
    K = 64
    s = (2.0 ** rng.integers(-3, 4, size=K)).astype(np.float32)
    X = (rng.standard_normal((8, K)) * 2).astype(np.float16)
    W = (rng.standard_normal((12, K)) * 0.05).astype(np.float16)
    Xq, sx = nx.smooth_quantize_activations(X, s)
    Xq_b, sx_b = oracle.quantize_activations((X.astype(np.float32) / s).astype(np.float16),
                                             np.zeros(K, np.uint8))
    assert np.array_equal(Xq, Xq_b) and np.array_equal(sx, sx_b)
    Wq, sw = nx.smooth_quantize_weight(W, s)
    Wq_b, sw_b = oracle.quantize_weight((W.astype(np.float32) * s).astype(np.float16))
    assert np.array_equal(Wq, Wq_b) and np.array_equal(sw, sw_b)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_smoothquant_error_bound_against_fp64(nx, seed):
    """|Y - X W^T| within the closed-form bound of per-row / per-channel int8 on
    the smoothed operands (c = 1/2 + 127 * 2^-24 as for the int8 oracle), plus
    the 2^-23 relative move of the transform and half an fp16 ulp.  A product
    form of the factor would not balance the outlier channels and is caught
    by the balance pin; here a negative control without smoothing shows the
    bound is tight enough to matter on outlier data."""
    T, K, N = 9, 192, 21
    X, _ = synth.make_activations(T, K, seed=40 + seed, n_dims=4, mag=(20.0, 80.0))
    W = synth.make_weight(N, K, seed=40 + seed, sigma=0.04)
    s = nx.smooth_factors(nx.column_absmax(X), nx.column_absmax(W), 0.5)
    Wq, sw = nx.smooth_quantize_weight(W, s)
    Y = nx.smoothquant_matmul(X, s, Wq, sw).astype(np.float64)
    Xs, Ws = [a.astype(np.float64) for a in smoothed(X, W, s)]
    exact = X.astype(np.float64) @ W.astype(np.float64).T
    sx_ref = np.abs(Xs).max(axis=1) / 127.0
    sw_ref = np.abs(Ws).max(axis=1) / 127.0
    c = 0.5 + 127 * 2.0 ** -24
    bound = np.abs(Xs).sum(axis=1)[:, None] * sw_ref[None, :] * c \
        + sx_ref[:, None] * np.abs(Ws).sum(axis=1)[None, :] * c + K * sx_ref[:, None] * sw_ref[None, :] * c * c
    bound += 2.0 ** -22 * (np.abs(X.astype(np.float64)) @ np.abs(W.astype(np.float64)).T)
    bound = bound * (1 + 1e-6) + ulp16(exact) / 2 + 1e-12
    assert np.all(np.abs(Y - exact) <= bound)
    # smoothing matters here: plain per-row int8 of the unsmoothed X is worse
    ones = np.ones(K, np.float32)
    Wq1, sw1 = nx.smooth_quantize_weight(W, ones)
    Y1 = nx.smoothquant_matmul(X, ones, Wq1, sw1).astype(np.float64)
    assert np.abs(Y1 - exact).max() > 1.5 * np.abs(Y - exact).max()


# =================================================================== FP8 E4M3

def test_e4m3_code_table(nx):
    """The E4M3 format (1 sign, 4 exponent, 3 mantissa bits, bias 7, no
    infinities): largest finite 448 = 1.75 * 2^8 (code 0x7e), smallest normal
    2^-6 (code 0x08), smallest subnormal 2^-9 (code 0x01), 0x7f is NaN; the
    positive finite codes increase strictly; negatives mirror them."""
    v = nx.e4m3_to_float(np.arange(256))
    assert v[0x7e] == 448.0 and v[0x08] == 2.0 ** -6 and v[0x01] == 2.0 ** -9 and v[0] == 0.0
    assert np.isnan(v[0x7f]) and np.isnan(v[0xff])
    assert np.all(np.diff(v[:0x7f]) > 0)
    assert np.array_equal(v[0x80:0xff], -v[:0x7f])
    assert np.signbit(v[0x80])


def test_e4m3_encode_round_trip_and_ties(nx):
    v = nx.e4m3_to_float(np.arange(0x7f)).astype(np.float64)
    codes = np.arange(0x7f, dtype=np.uint8)
    assert np.array_equal(nx.float_to_e4m3(v), codes)                      # every finite code
    assert np.array_equal(nx.float_to_e4m3(-v), codes | 0x80)             # and its negative
    mid = (v[:-1] + v[1:]) / 2                                             # exact in binary32
    even = np.where(codes[:-1] % 2 == 0, codes[:-1], codes[1:])
    assert np.array_equal(nx.float_to_e4m3(mid), even)                     # ties to even
    assert np.array_equal(nx.float_to_e4m3(np.nextafter(mid.astype(np.float32), np.float32(0))), codes[:-1])
    assert np.array_equal(nx.float_to_e4m3(np.nextafter(mid.astype(np.float32), np.float32(1e9))), codes[1:])
    assert nx.float_to_e4m3(np.array([449.0, 464.0, 1e6], np.float32)).tolist() == [0x7e] * 3  # saturate
    assert nx.float_to_e4m3(np.array([-0.0, -2.0 ** -11], np.float32)).tolist() == [0x80, 0x80]


def test_e4m3_encode_matches_torch(nx):
    """torch's float8_e4m3fn cast (round to nearest even) on a dense grid of
    binary32 values inside the finite range."""
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(6)
    x = np.concatenate([rng.uniform(-448, 448, 4000), rng.uniform(-1, 1, 4000) * 2.0 ** -5,
                        rng.uniform(-2, 2, 4000)]).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(nx.float_to_e4m3(x), ref)


def test_fp8_weight_codes_reach_448_at_the_row_maximum(nx):
    W = synth.make_weight(20, 64, seed=7, sigma=0.05)
    W[3] = 0
    Wq, sw = nx.fp8_quantize_weight(W)
    Wd = W.astype(np.float32)
    assert np.array_equal(sw, (np.abs(Wd).max(axis=1) / np.float32(448.0)).astype(np.float32))
    am = np.abs(Wd).argmax(axis=1)
    for n in range(20):
        if n == 3:
            assert sw[n] == 0 and not Wq[n].any()
        else:
            assert Wq[n, am[n]] & 0x7f == 0x7e


def test_fp8_gemm_is_exact(nx):
    rng = np.random.default_rng(8)
    A = rng.integers(0, 256, size=(5, 300)).astype(np.uint8)
    B = rng.integers(0, 256, size=(7, 300)).astype(np.uint8)
    A[(A & 0x7f) == 0x7f] = 0     # no NaN codes
    B[(B & 0x7f) == 0x7f] = 0
    ref = nx.e4m3_to_float(A).astype(np.float64) @ nx.e4m3_to_float(B).astype(np.float64).T
    assert np.array_equal(nx.fp8_gemm(A, B), ref)


def test_fp8_tau_zero_is_fp16_gemm(nx):
    X, W = synth.random_case(6, 96, 11, seed=9)
    Wq, sw = nx.fp8_quantize_weight(W)
    Y = nx.fp8_matmul(X, Wq, sw, W, 0.0)
    exact = X.astype(np.float64) @ W.astype(np.float64).T
    assert np.all(np.abs(Y.astype(np.float64) - exact) <= ulp16(exact) / 2)


def test_fp8_representable_inputs_quantise_exactly(nx):
    """Rows made of E4M3 values times a power of two, each reaching 448 times
    that power: scale and codes are exact, so Y = fp16(X W^T)."""
    rng = np.random.default_rng(10)
    vals = nx.e4m3_to_float(np.arange(0x7f)).astype(np.float64)
    vals = vals[vals >= 2.0 ** -3]                      # stay clear of fp16 subnormals after scaling

    def rows(n, K, e):
        r = rng.choice(vals, size=(n, K)) * np.where(rng.random((n, K)) < 0.5, -1, 1)
        r[np.arange(n), rng.integers(0, K, n)] = 448.0
        return (r * 2.0 ** e).astype(np.float16)
    X, W = rows(5, 48, -6), rows(9, 48, -10)
    Wq, sw = nx.fp8_quantize_weight(W)
    Y = nx.fp8_matmul(X, Wq, sw, W, float("inf"))
    exact = X.astype(np.float64) @ W.astype(np.float64).T
    assert np.all(np.abs(Y.astype(np.float64) - exact) <= ulp16(exact) / 2)


@pytest.mark.parametrize("seed", [0, 1])
def test_fp8_error_bound_against_fp64(nx, seed):
    """Each regular element: |x - s e4m3(x/s)| <= |x| 2^-4 + s 2^-10 (half a
    3-bit-mantissa ulp, or half the subnormal step 2^-9), with 2^-23 of slack
    for the binary32 division; the outlier part is exact.  A worst-case bound:
    mistakes in the codes themselves are caught by the code-table, rounding,
    scale and exactly-representable pins above."""
    T, K, N = 7, 160, 15
    X, W = synth.random_case(T, K, N, seed=50 + seed, n_dims=3, mag=(8.0, 60.0))
    Wq, sw = nx.fp8_quantize_weight(W)
    Y = nx.fp8_matmul(X, Wq, sw, W, 6.0).astype(np.float64)
    Xd, Wd = X.astype(np.float64), W.astype(np.float64)
    exact = Xd @ Wd.T
    R = ~np.any(np.abs(Xd) >= 6.0, axis=0)
    sx_ref = np.abs(Xd[:, R]).max(axis=1) / 448.0
    sw_ref = np.abs(Wd).max(axis=1) / 448.0
    e = 2.0 ** -4 + 2.0 ** -23
    dx = np.abs(Xd[:, R]) * e + sx_ref[:, None] * 2.0 ** -10     # [T, |R|]
    dw = np.abs(Wd[:, R]) * e + sw_ref[:, None] * 2.0 ** -10     # [N, |R|]
    bound = dx @ (np.abs(Wd[:, R]) + dw).T + np.abs(Xd[:, R]) @ dw.T
    bound = bound * (1 + 1e-6) + ulp16(exact) / 2 + 1e-12
    assert np.all(np.abs(Y - exact) <= bound)


# =================================================================== stored outlier columns

def test_reconstructed_weight_is_the_fp16_of_the_binary32_product(nx):
    rng = np.random.default_rng(11)
    for _ in range(2000):
        q = int(rng.integers(-127, 128))
        s = np.float32(abs(rng.standard_normal()) * 10.0 ** rng.integers(-4, 1))
        want = np.float16(np.float32(s) * np.float32(q))
        got = nx.reconstruct_weight(q, s)
        assert got.view(np.uint16) == want.view(np.uint16), (q, s)


def test_reconstruction_rounds_twice(nx):
    """The product is rounded to binary32 first, then to fp16: where the exact
    product sits just above an fp16 half-way point but its binary32 rounding
    lands on it, ties-to-even takes the lower neighbour (one rounding of the
    exact product would take the upper one)."""
    found = 0
    for q in (3, 5, 7, 9, 11, 13, 101, 127):
        for h in range(0x3c01, 0x3c80, 2):                       # fp16 values in [1, 1.25), odd mantissa
            lo = np.uint16(h - 1).view(np.float16)                 # even neighbour below
            hi = np.uint16(h).view(np.float16)
            m = (Fraction(float(lo)) + Fraction(float(hi))) / 2   # the half-way point
            s = np.float32(float(m) / q)
            for _ in range(4):
                exact = Fraction(float(s)) * q
                if exact > m and np.float32(float(s) * q) == np.float32(float(m)):
                    got = nx.reconstruct_weight(q, s)
                    assert got.view(np.uint16) == lo.view(np.uint16), (q, h)
                    found += 1
                    break
                s = np.nextafter(s, np.float32(1))
    assert found >= 5


def test_full_store_equals_the_fp16_weight(nx, oracle):
    X, W = synth.random_case(10, 128, 37, seed=12, n_dims=5)
    Wq, sw = oracle.quantize_weight(W)
    slot, Wst = nx.make_store(W, np.arange(128))
    for tau in (6.0, 0.0, float("inf")):
        Y, miss = nx.matmul_stored(X, Wq, sw, slot, Wst, tau)
        assert miss == 0
        assert np.array_equal(Y.view(np.uint16), oracle.matmul(X, Wq, sw, W, tau).view(np.uint16))


def test_empty_store_on_exactly_reconstructible_weights(nx, oracle):
    """Weights q * 2^-7 with each row reaching |q| = 127: sw = 2^-7 and every
    reconstruction fp16(sw q) is the weight itself, so a store with no columns
    gives the fp16-weight result bit for bit, and every outlier is a miss."""
    rng = np.random.default_rng(13)
    N, K = 19, 96
    q = rng.integers(-127, 128, size=(N, K))
    q[np.arange(N), rng.integers(0, K, N)] = 127
    W = (q * 2.0 ** -7).astype(np.float16)
    Wq, sw = oracle.quantize_weight(W)
    assert np.all(sw == np.float32(2.0 ** -7)) and np.array_equal(Wq, q.astype(np.int8))
    X, _ = synth.make_activations(8, K, seed=13, n_dims=4, mag=(8.0, 40.0))
    slot, Wst = nx.make_store(W, [])
    Y, miss = nx.matmul_stored(X, Wq, sw, slot, Wst, 6.0)
    assert miss == oracle.compact(oracle.detect_outliers(X, 6.0)).size == 4
    assert np.array_equal(Y.view(np.uint16), oracle.matmul(X, Wq, sw, W, 6.0).view(np.uint16))


def test_partial_store_outlier_part_by_exact_rationals(nx, oracle):
    X, W = synth.random_case(3, 32, 4, seed=14, n_dims=5, mag=(8.0, 30.0))
    Wq, sw = oracle.quantize_weight(W)
    idx = oracle.compact(oracle.detect_outliers(X, 6.0))
    assert idx.size == 5
    stored = idx[::2]
    slot, Wst = nx.make_store(W, stored)
    yo, miss = nx.outlier_gemm_stored(X, Wq, sw, slot, Wst, idx)
    assert miss == idx.size - stored.size
    for t in range(3):
        for n in range(4):
            ref = Fraction(0)
            for k in idx:
                if k in stored:
                    w = Fraction(float(W[n, k]))
                else:
                    w = Fraction(float(np.float16(np.float32(sw[n]) * np.float32(Wq[n, k]))))
                ref += Fraction(float(X[t, k])) * w
            assert abs(Fraction(yo[t, n]) - ref) <= abs(ref) * Fraction(1, 2 ** 50) + Fraction(1, 2 ** 80)
