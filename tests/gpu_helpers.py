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
