"""GPU parity of the LLM.int8() matmul reading its fp16 outlier weights from a
column store instead of the full fp16 weight (through the C ABI), against the
CPU oracle.

The store itself (slot map and fp16 columns) and the int32 accumulator bit for
bit; the miss count exactly; Y within |Y_gpu - Y_oracle| <= 1e-3 max|Y_oracle|
+ 1 fp16 ulp.  With every column stored, Y must equal the fp16-weight entry
bit for bit (the same fp16 values reach the same kernels).
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


def test_store_build_bitexact(L, nx):
    W = synth.make_weight(1000, 1040, seed=1)
    cols = np.random.default_rng(1).choice(1040, size=37, replace=False).astype(np.int32)
    slot, Wst = L.llmint8_outlier_store_build(dev(W), dev(cols))
    slot_o, Wst_o = nx.make_store(W, cols)
    torch.cuda.synchronize()
    assert L.llmint8_sync_status() == 0
    assert_equal(host(slot), slot_o, "slot")
    assert_equal(host(Wst).view(np.uint16), Wst_o.view(np.uint16), "stored columns")


def test_store_build_rejects_a_column_outside_k(L):
    """A column index past K is skipped by the build kernel (no access is made
    with it) and reported on the host."""
    W = torch.zeros((64, 256), dtype=torch.float16, device="cuda")
    L.llmint8_outlier_store_build(W, torch.tensor([3, 256 + 5], dtype=torch.int32, device="cuda"))
    assert L.llmint8_sync_status() == L.llmint8.LLMINT8_ERR_INVALID_ARG
    assert L.llmint8_sync_status() == 0


def run_stored(L, nx, oracle, X, W, cols, tau, path, expect_bitwise_with_w=False):
    T, K = X.shape
    N = W.shape[0]
    cols = np.asarray(cols, dtype=np.int32)
    Wq_o, sw_o = oracle.quantize_weight(W)
    slot_o, Wst_o = nx.make_store(W, cols)
    Y_o, miss_o = nx.matmul_stored(X, Wq_o, sw_o, slot_o, Wst_o, tau)
    flag = oracle.detect_outliers(X, tau)
    Xq_o, _ = oracle.quantize_activations(X, flag)
    acc_o = oracle.int8_gemm(Xq_o, Wq_o)
    Wd = dev(W)
    Wq, sw = L.llmint8_quantize_weight(Wd)
    slot, Wst = L.llmint8_outlier_store_build(Wd, dev(cols))
    miss = torch.full((1,), -7, dtype=torch.int32, device="cuda")
    acc = torch.empty((T, N), dtype=torch.int32, device="cuda")
    Xd = dev(X)
    Y = L.llmint8_matmul_stored(Xd, Wq, sw, slot, Wst, tau, n_miss=miss, path=path, acc_out=acc)
    Yw = L.llmint8_matmul_debug(Xd, Wq, sw, Wd, tau, path=path) if expect_bitwise_with_w else None
    torch.cuda.synchronize()
    assert L.llmint8_sync_status() == 0
    assert int(host(miss)[0]) == miss_o, (int(host(miss)[0]), miss_o)
    assert_equal(host(acc), acc_o, "acc")
    assert_y_close(host(Y), Y_o, "Y")
    if Yw is not None:
        assert_equal(host(Y).view(np.uint16), host(Yw).view(np.uint16), "full store vs fp16 weight")
    return miss_o


CASES = [(1, 1, 300, 256), (1, 7, 1000, 1040), (1, 16, 11008, 4096), (2, 17, 300, 272), (2, 129, 513, 1040),
         (2, 300, 1000, 4096)]


@pytest.mark.parametrize("path,T,N,K", CASES)
def test_full_store_equals_fp16_weight(L, nx, oracle, path, T, N, K):
    X, W = synth.random_case(T, K, N, seed=T + N + K, n_dims=min(5, K), mag=(6.0, 50.0))
    for tau in (6.0, 0.0):
        run_stored(L, nx, oracle, X, W, np.arange(K), tau, path, expect_bitwise_with_w=True)


@pytest.mark.parametrize("path,T,N,K", CASES)
def test_partial_and_empty_store(L, nx, oracle, path, T, N, K):
    X, W = synth.random_case(T, K, N, seed=2 * T + N + K, n_dims=min(6, K), mag=(6.0, 50.0))
    idx = oracle.compact(oracle.detect_outliers(X, 6.0))
    partial = np.concatenate([idx[::2], np.arange(0, K, 97)])
    partial = np.unique(partial)
    assert run_stored(L, nx, oracle, X, W, partial, 6.0, path) == np.setdiff1d(idx, partial).size
    assert run_stored(L, nx, oracle, X, W, [], 6.0, path) == idx.size
    run_stored(L, nx, oracle, X, W, [], 0.0, path)      # every column an outlier, none stored


@pytest.mark.parametrize("name", ["7b_decode", "7b_prefill", "13b_up"])
def test_store_full_size(L, nx, oracle, name):
    """The workloads with the store holding their systematic outlier dims (what
    a calibration batch finds); the 7B prefill's random spike columns are
    misses."""
    w = synth.workload(name)
    miss = run_stored(L, nx, oracle, w["X"], w["W"], np.sort(w["dims"]), 6.0, 0)
    if name == "7b_prefill":
        assert miss > 0
    else:
        assert miss == 0


def test_int8_linear_with_a_store_drops_the_fp16_weight(L, nx, oracle):
    X, W = synth.random_case(40, 512, 96, seed=10, n_dims=4)
    idx = oracle.compact(oracle.detect_outliers(X, 6.0))
    lin = L.Int8Linear(dev(W), store_columns=idx[:-1])
    assert lin.W is None
    assert lin.resident_weight_bytes() == 96 * 512 + 4 * 96 + 2 * 96 * (idx.size - 1) + 4 * 512
    Y = lin(dev(X))
    torch.cuda.synchronize()
    assert lin.last_misses == 1
    Wq_o, sw_o = oracle.quantize_weight(W)
    slot_o, Wst_o = nx.make_store(W, idx[:-1])
    Y_o, miss = nx.matmul_stored(X, Wq_o, sw_o, slot_o, Wst_o, 6.0)
    assert miss == 1
    assert_y_close(host(Y), Y_o, "Y")
