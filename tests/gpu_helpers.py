"""Shared helpers of the GPU parity tests (imports torch lazily)."""
import numpy as np


def ulp16(y):
    y = np.abs(np.asarray(y, dtype=np.float64))
    e = np.floor(np.log2(np.maximum(y, 2.0 ** -14)))
    return 2.0 ** (e - 10)


def assert_y_close(y_gpu, y_ref, what=""):
    """|Y_gpu - Y_oracle| <= 1e-3 * max|Y_oracle| + 1 fp16 ulp(Y_oracle), elementwise."""
    g = np.asarray(y_gpu, dtype=np.float64)
    r = np.asarray(y_ref, dtype=np.float64)
    assert g.shape == r.shape, (g.shape, r.shape)
    assert np.all(np.isfinite(r)), "oracle result not finite"
    tol = 1e-3 * (np.abs(r).max() if r.size else 0.0) + ulp16(r)
    err = np.abs(g - r)
    bad = ~(err <= tol)
    if bad.any():
        i = np.unravel_index(np.argmax(np.where(bad, err - tol, -np.inf)), err.shape)
        raise AssertionError(f"{what}: {int(bad.sum())}/{bad.size} outside tolerance; worst at "
                             f"{i}: gpu={g[i]} oracle={r[i]} tol={tol[i]}")


def assert_equal(a, b, what=""):
    a = np.asarray(a)
    b = np.asarray(b)
    assert a.shape == b.shape, (what, a.shape, b.shape)
    if not np.array_equal(a, b):
        d = np.argwhere(a != b)
        raise AssertionError(f"{what}: {len(d)} mismatches, first at {tuple(d[0])}: "
                             f"{a[tuple(d[0])]} vs {b[tuple(d[0])]}")


def projected_weights(Wq_o, vectors=4, seed=0, chunk=4096):
    """(r, Wq_o^T r) for `vectors` random integer columns r in [-1024, 1024]^N.
    The product is summed in binary64, where every partial sum is an integer
    of magnitude <= 127 * 1024 * N < 2^53 and so exact in any order; returned
    as int64."""
    N, K = Wq_o.shape
    assert 127 * 1024 * N < 2 ** 53
    r = np.random.default_rng(seed).integers(-1024, 1025, size=(N, vectors)).astype(np.int64)
    wr = np.zeros((K, vectors), np.float64)
    rf = r.astype(np.float64)
    for n0 in range(0, N, chunk):
        wr += Wq_o[n0:n0 + chunk].astype(np.float64).T @ rf[n0:n0 + chunk]
    return r, wr.astype(np.int64)


def assert_acc_exact(acc, Xq_o, projection, what="", chunk=512):
    """Every element of an int32 [T, N] accumulator against Xq_o Wq_o^T without
    forming the product (Freivalds' check): acc r == Xq_o (Wq_o^T r) exactly in
    int64 for each random column r of `projection` (from projected_weights).
    A row of acc with any wrong element passes one column with probability at
    most 1/2049 (at most one of the 2049 values of one coordinate of r zeroes
    the row's error against r).  int64 is exact while K * 127 * 127 * 1024 * N
    stays below 2^63."""
    r, wr = projection
    acc = np.asarray(acc)
    T, N = acc.shape
    assert Xq_o.shape[0] == T and r.shape[0] == N, (acc.shape, Xq_o.shape, r.shape)
    for t0 in range(0, T, chunk):
        lhs = acc[t0:t0 + chunk].astype(np.int64) @ r
        rhs = Xq_o[t0:t0 + chunk].astype(np.int64) @ wr
        if not np.array_equal(lhs, rhs):
            bad = np.nonzero((lhs != rhs).any(axis=1))[0] + t0
            raise AssertionError(f"{what}: acc differs from Xq Wq^T in {bad.size} rows, "
                                 f"first {bad[:8].tolist()}")
