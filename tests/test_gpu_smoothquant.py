"""GPU parity of SmoothQuant W8A8 (through the C ABI) against the CPU oracle.

Channel maxima, smoothing factors (alpha 0, 1/2, 1), smoothed weight codes and
scales, activation codes and scales and the int32 accumulator bit for bit; Y
within |Y_gpu - Y_oracle| <= 1e-3 max|Y_oracle| + 1 fp16 ulp.  The factors
given to the matmul are the oracle's, so both sides quantise the same values.
"""
import numpy as np
import pytest

from gpu_helpers import assert_equal, assert_y_close
from int8_mixed_precision_outlier_b200 import synth

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def L():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from int8_mixed_precision_outlier_b200 import _build
    _build.build()
    import int8_mixed_precision_outlier_b200 as L
    L.load_library()
    return L


@pytest.fixture(scope="module")
def nx():
    from oracle import oracle_next as O
    O.build()
    return O


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def host(t):
    return t.detach().cpu().numpy()


def bits(a):
    return np.ascontiguousarray(a).view(np.uint32)


@pytest.mark.parametrize("rows,K", [(1, 16), (7, 272), (300, 1040), (2048, 4096), (5, 8192)])
def test_column_absmax_bitexact(L, nx, rows, K):
    A, _ = synth.make_activations(rows, K, seed=rows + K, n_dims=min(4, K), mag=(6.0, 90.0))
    amax = L.llmint8_column_absmax(dev(A))
    torch.cuda.synchronize()
    assert_equal(bits(host(amax)), bits(nx.column_absmax(A)), "column maxima")


def test_column_absmax_accumulates_batches(L, nx):
    A1, _ = synth.make_activations(40, 512, seed=1, n_dims=3, mag=(6.0, 50.0))
    A2, _ = synth.make_activations(33, 512, seed=2, n_dims=3, mag=(6.0, 80.0))
    amax = L.llmint8_column_absmax(dev(A1))
    L.llmint8_column_absmax(dev(A2), amax, accumulate=True)
    torch.cuda.synchronize()
    assert_equal(bits(host(amax)), bits(nx.column_absmax(np.concatenate([A1, A2]))), "two batches")


@pytest.mark.parametrize("alpha", [0.5, 1.0, 0.0, 0.3, 0.75])
def test_smooth_factors(L, nx, alpha):
    rng = np.random.default_rng(3)
    ax = (rng.random(4096) * 100).astype(np.float32)
    aw = (rng.random(4096) * 0.1).astype(np.float32)
    ax[:3] = 0.0
    aw[5:7] = 0.0
    s = host(L.llmint8_smooth_factors(dev(ax), dev(aw), alpha))
    s_o = nx.smooth_factors(ax, aw, alpha)
    if alpha in (0.5, 1.0, 0.0):
        assert_equal(bits(s), bits(s_o), f"factors alpha={alpha}")
    else:   # powf on both sides: a few ulps apart at most
        assert np.all(np.abs(s.astype(np.float64) - s_o) <= 4 * 2.0 ** -23 * np.abs(s_o))
    assert np.all(s[:3] == 1.0) and np.all(s[5:7] == 1.0)


def oracle_factors(nx, X, W, alpha=0.5):
    return nx.smooth_factors(nx.column_absmax(X), nx.column_absmax(W), alpha)


@pytest.mark.parametrize("N,K", [(1, 16), (300, 1040), (513, 4096)])
def test_smoothquant_weight_bitexact(L, nx, N, K):
    X, W = synth.random_case(64, K, N, seed=N + K, n_dims=min(4, K), mag=(8.0, 60.0))
    W[0, :2] = 0
    s = oracle_factors(nx, X, W)
    Wq, sw = L.llmint8_smoothquant_quantize_weight(dev(W), dev(s))
    Wq_o, sw_o = nx.smooth_quantize_weight(W, s)
    torch.cuda.synchronize()
    assert_equal(host(Wq), Wq_o, "Wq")
    assert_equal(bits(host(sw)), bits(sw_o), "Wscale")


def run_smoothquant(L, nx, oracle, X, W, path, alpha=0.5):
    T, K = X.shape
    N = W.shape[0]
    s = oracle_factors(nx, X, W, alpha)
    Wq_o, sw_o = nx.smooth_quantize_weight(W, s)
    Y_o, im = nx.smoothquant_matmul(X, s, Wq_o, sw_o, intermediates=True)
    sd = dev(s)
    Wq, sw = L.llmint8_smoothquant_quantize_weight(dev(W), sd)
    acc = torch.empty((T, N), dtype=torch.int32, device="cuda")
    Xq = torch.empty((T, K), dtype=torch.int8, device="cuda")
    sx = torch.empty(T, dtype=torch.float32, device="cuda")
    Y = L.llmint8_smoothquant_matmul(dev(X), sd, Wq, sw, path=path, acc_out=acc, xq_out=Xq, sx_out=sx)
    Y2 = L.llmint8_smoothquant_matmul(dev(X), sd, Wq, sw)   # plain entry, same kernels for these shapes
    torch.cuda.synchronize()
    assert L.llmint8_sync_status() == 0
    assert_equal(host(Wq), Wq_o, "Wq")
    assert_equal(bits(host(sw)), bits(sw_o), "Wscale")
    assert_equal(host(Xq), im["Xq"], "Xq")
    assert_equal(bits(host(sx)), bits(im["sx"]), "sx")
    assert_equal(host(acc), im["acc"], "acc")
    assert_y_close(host(Y), Y_o, "Y")
    assert_equal(host(Y2).view(np.uint16), host(Y).view(np.uint16), "plain and inspection entries")


@pytest.mark.parametrize("path,T,N,K", [(1, 1, 300, 256), (1, 16, 1000, 1040), (1, 5, 11008, 4096),
                                        (2, 17, 300, 272), (2, 129, 513, 1040), (2, 300, 1000, 4096),
                                        (2, 600, 20000, 1024)])
def test_smoothquant_matmul(L, nx, oracle, path, T, N, K):
    X, W = synth.random_case(T, K, N, seed=T + N + K, n_dims=min(5, K), mag=(8.0, 60.0))
    run_smoothquant(L, nx, oracle, X, W, path)


@pytest.mark.parametrize("name", ["7b_prefill", "13b_up"])
def test_smoothquant_full_size(L, nx, oracle, name):
    """The 7B prefill and 13B up-projection workloads, every element; the
    factors come from the workload's own activations (calibration = input)."""
    w = synth.workload(name)
    run_smoothquant(L, nx, oracle, w["X"], w["W"], 0)
