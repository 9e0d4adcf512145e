"""The host-side checks the GPU parity tests rely on, exercised on the CPU
against the oracle: the projection check of a full int32 accumulator passes
on the exact product and catches planted single-element errors."""
import numpy as np
import pytest

from gpu_helpers import assert_acc_exact, projected_weights
from int8_mixed_precision_outlier_b200 import synth


@pytest.fixture(scope="module")
def case(oracle):
    X, W = synth.random_case(97, 1040, 700, seed=31, n_dims=4, mag=(6.0, 50.0))
    Wq, _ = oracle.quantize_weight(W)
    Xq, _ = oracle.quantize_activations(X, oracle.detect_outliers(X, 6.0))
    return Xq, Wq, oracle.int8_gemm(Xq, Wq)


def test_projection_check_passes_on_the_exact_product(case):
    Xq, Wq, acc = case
    assert_acc_exact(acc, Xq, projected_weights(Wq, seed=5), "exact")


@pytest.mark.parametrize("t,n,delta", [(0, 0, 1), (96, 699, -1), (40, 350, 2 ** 20), (13, 77, -7)])
def test_projection_check_catches_one_wrong_element(case, t, n, delta):
    Xq, Wq, acc = case
    bad = acc.copy()
    bad[t, n] += delta
    with pytest.raises(AssertionError, match=rf"first \[{t}\]"):
        assert_acc_exact(bad, Xq, projected_weights(Wq, seed=5), "planted")


def test_projection_check_catches_swapped_rows(case):
    Xq, Wq, acc = case
    bad = acc.copy()
    bad[[3, 4]] = bad[[4, 3]]
    with pytest.raises(AssertionError):
        assert_acc_exact(bad, Xq, projected_weights(Wq, seed=5), "swapped")


def test_projection_is_exact_against_int64(case):
    _, Wq, _ = case
    r, wr = projected_weights(Wq, seed=9)
    assert np.array_equal(wr, Wq.astype(np.int64).T @ r)
