"""GPU parity of the FP8 (E4M3) decomposition (through the C ABI) against the
CPU oracle.

The E4M3 weight and activation codes, their scales and the outlier list must
match bit for bit.  The f32 accumulator of the E4M3 products is a floating-
point sum (the oracle's binary64 sum is exact): it is held to the recursive
summation bound, |acc - exact| <= K * 2^-23 * sum_k |x_k w_k|, and Y to the
tolerance of every other test, |Y_gpu - Y_oracle| <= 1e-3 max|Y_oracle| + 1
fp16 ulp.
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


def test_fp8_weight_codes_every_fp16_value(L, nx):
    """Every finite fp16 bit pattern as a weight element, under many row
    scales: the conversions (binary32 quotient, round to nearest even,
    saturation, signed zeros, subnormal codes) agree bit for bit."""
    pos = np.arange(0, 0x7c00, dtype=np.uint16)
    vals = np.concatenate([pos, pos | 0x8000]).view(np.float16)           # 63488 values, +-0 included
    K = 256
    rows = vals[: (vals.size // K) * K].reshape(-1, K).copy()
    rng = np.random.default_rng(0)
    rows = rows[rng.permutation(rows.shape[0])]
    Wq, sw = L.llmint8_fp8_quantize_weight(dev(rows))
    Wq_o, sw_o = nx.fp8_quantize_weight(rows)
    torch.cuda.synchronize()
    assert_equal(bits(host(sw)), bits(sw_o), "scales")
    assert_equal(host(Wq), Wq_o, "E4M3 codes")


@pytest.mark.parametrize("N,K", [(1, 16), (300, 1040), (513, 4096)])
def test_fp8_weight_codes_bitexact(L, nx, N, K):
    W = synth.make_weight(N, K, seed=N + K, sigma=0.05)
    W[0, :3] = 0
    Wq, sw = L.llmint8_fp8_quantize_weight(dev(W))
    Wq_o, sw_o = nx.fp8_quantize_weight(W)
    torch.cuda.synchronize()
    assert_equal(host(Wq), Wq_o, "Wq")
    assert_equal(bits(host(sw)), bits(sw_o), "Wscale")


def acc_bound(nx, Xq, Wq):
    """K * 2^-23 * sum_k |x_k w_k| from the decoded codes (binary64, exact)."""
    a = np.abs(nx.e4m3_to_float(Xq).astype(np.float64))
    b = np.abs(nx.e4m3_to_float(Wq).astype(np.float64))
    return Xq.shape[1] * 2.0 ** -23 * (a @ b.T)


def run_fp8(L, nx, X, W, tau, path, check_acc=True):
    T, K = X.shape
    N = W.shape[0]
    Wq_o, sw_o = nx.fp8_quantize_weight(W)
    Y_o, im = nx.fp8_matmul(X, Wq_o, sw_o, W, tau, intermediates=True)
    Wd = dev(W)
    Wq, sw = L.llmint8_fp8_quantize_weight(Wd)
    acc = torch.empty((T, N), dtype=torch.float32, device="cuda")
    Xq = torch.empty((T, K), dtype=torch.uint8, device="cuda")
    sx = torch.empty(T, dtype=torch.float32, device="cuda")
    idx = torch.empty(K, dtype=torch.int32, device="cuda")
    n = torch.zeros(1, dtype=torch.int32, device="cuda")
    Xd = dev(X)
    Y = L.llmint8_fp8_matmul(Xd, Wq, sw, Wd, tau, path=path, acc_out=acc, xq_out=Xq, sx_out=sx, idx_out=idx,
                             n_out=n)
    Y2 = L.llmint8_fp8_matmul(Xd, Wq, sw, Wd, tau, path=path)
    torch.cuda.synchronize()
    assert L.llmint8_sync_status() == 0
    assert_equal(host(Wq), Wq_o, "Wq")
    assert_equal(bits(host(sw)), bits(sw_o), "Wscale")
    assert_equal(host(idx)[: int(host(n)[0])], im["idx"], "outlier idx")
    assert_equal(host(Xq), im["Xq"], "Xq")
    assert_equal(bits(host(sx)), bits(im["sx"]), "sx")
    if check_acc:
        err = np.abs(host(acc).astype(np.float64) - im["acc"])
        assert np.all(err <= acc_bound(nx, im["Xq"], Wq_o)), f"acc error {err.max()}"
    assert_y_close(host(Y), Y_o, "Y")
    assert_equal(host(Y2).view(np.uint16), host(Y).view(np.uint16), "with and without inspection outputs")


SMALL = [(1, 1, 128, 256), (1, 3, 300, 272), (1, 16, 1000, 1024), (1, 16, 11008, 4096), (2, 1, 256, 256),
         (2, 17, 300, 272), (2, 129, 513, 1040), (2, 300, 1000, 1024), (2, 600, 20000, 1024)]


@pytest.mark.parametrize("path,T,N,K", SMALL)
@pytest.mark.parametrize("tau", [6.0, float("inf"), 0.0])
def test_fp8_matmul(L, nx, path, T, N, K, tau):
    X, W = synth.random_case(T, K, N, seed=T + N + K, n_dims=min(5, K), mag=(6.0, 50.0))
    run_fp8(L, nx, X, W, tau, path)


@pytest.mark.parametrize("name", ["7b_prefill", "13b_up"])
def test_fp8_full_size(L, nx, name):
    """The 7B prefill and 13B up-projection workloads, every element."""
    w = synth.workload(name)
    run_fp8(L, nx, w["X"], w["W"], 6.0, 0, check_acc=False)


def test_fp8_decode_7b(L, nx):
    w = synth.workload("7b_decode")
    for T in (1, 4, 16):
        run_fp8(L, nx, np.ascontiguousarray(w["X"][:T]), w["W"], 6.0, 0)
