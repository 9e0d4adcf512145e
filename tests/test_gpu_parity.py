"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle.

Integer stages (Wq, Wscale, outlier set, Xq, sx, int32 acc) must match bit for
bit; Y must satisfy |Y_gpu - Y_oracle| <= 1e-3 max|Y_oracle| + 1 fp16 ulp.
Every case compares every element, the full-size workloads (7B prefill, 13B
up-projection, 70B up-projection at thresholds 4, 6 and inf) included: there a
projection check of the int32 accumulator runs first as a quick filter, then
the oracle's full int8 product and fp part.
"""
import numpy as np
import pytest

from gpu_helpers import assert_acc_exact, assert_equal, assert_y_close, projected_weights
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


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def host(t):
    return t.detach().cpu().numpy()


def ok_status(L):
    assert L.llmint8_sync_status() == 0


def run_full(L, oracle, X, W, tau, path):
    """GPU and oracle on every element; returns nothing, asserts parity."""
    Wq_o, sw_o = oracle.quantize_weight(W)
    Y_o, im = oracle.matmul(X, Wq_o, sw_o, W, tau, intermediates=True)
    Xd, Wd = dev(X), dev(W)
    Wq, sw = L.llmint8_quantize_weight(Wd)
    Y, acc, Xq, sx, idx = L.llmint8_matmul_intermediates(Xd, Wq, sw, Wd, tau, path=path)
    Y2 = L.llmint8_matmul_debug(Xd, Wq, sw, Wd, tau, path=path)
    torch.cuda.synchronize()
    ok_status(L)
    assert_equal(host(Y2), host(Y), "with and without inspection outputs")
    assert_equal(host(Wq), Wq_o, "Wq")
    assert_equal(host(sw).view(np.uint32), sw_o.view(np.uint32), "Wscale")
    assert_equal(host(idx), im["idx"], "outlier idx")
    assert_equal(host(Xq), im["Xq"], "Xq")
    assert_equal(host(sx).view(np.uint32), im["sx"].view(np.uint32), "sx")
    assert_equal(host(acc), im["acc"], "acc")
    assert_y_close(host(Y), Y_o, "Y")


# --------------------------------------------------------------- weights

@pytest.mark.parametrize("N,K", [(1, 16), (3, 48), (256, 256), (301, 1040), (17, 4096)])
def test_quantize_weight_bitexact(L, oracle, N, K):
    W = synth.make_weight(N, K, seed=N + K, sigma=0.05)
    W[0, :3] = np.array([0.0, -0.0, 0.0], np.float16)
    Wq, sw = L.llmint8_quantize_weight(dev(W))
    Wq_o, sw_o = oracle.quantize_weight(W)
    assert_equal(host(Wq), Wq_o, "Wq")
    assert_equal(host(sw).view(np.uint32), sw_o.view(np.uint32), "Wscale")


def test_quantize_weight_worked_example_and_zero_row(L, oracle):
    from conftest import read_golden
    g = read_golden("worked_example_quant.txt")
    row = np.zeros(16, np.float32)
    row[:6] = [float(s) for s in g["input"]]
    W = np.stack([row, np.zeros(16, np.float32)]).astype(np.float16)
    Wq, sw = L.llmint8_quantize_weight(dev(W))
    assert host(Wq)[0, :6].tolist() == [int(s) for s in g["codes"]]
    assert host(sw)[1] == 0.0 and not host(Wq)[1].any()


# --------------------------------------------------------------- activations

def activation_stages(L, X, tau, path):
    """(Xq, sx, idx) of the given path, from the activation kernels alone and
    from inside a matmul call; the two must agree."""
    a = L.llmint8_detect_quantize(dev(X), tau, path=path)
    K = X.shape[1]
    W = torch.zeros((128, K), dtype=torch.float16, device="cuda")
    Wq, sw = L.llmint8_quantize_weight(W)
    _, _, Xq, sx, idx = L.llmint8_matmul_intermediates(dev(X), Wq, sw, W, tau, path=path)
    torch.cuda.synchronize()
    assert_equal(host(a[0]), host(Xq), "Xq alone vs in matmul")
    assert_equal(host(a[1]).view(np.uint32), host(sx).view(np.uint32), "sx alone vs in matmul")
    assert_equal(host(a[2]), host(idx), "idx alone vs in matmul")
    return Xq, sx, idx


@pytest.mark.parametrize("path,T", [(1, 1), (1, 5), (1, 16), (2, 1), (2, 17), (2, 130), (2, 300)])
@pytest.mark.parametrize("K", [16, 272, 1040, 4096])
def test_activation_stages_bitexact(L, oracle, path, T, K):
    X, _ = synth.make_activations(T, K, seed=T * 7 + K, n_dims=min(3, K), mag=(6.0, 60.0),
                                  spike_rate=2e-3)
    for tau in (6.0, float("inf"), 0.0, 2.5):
        Xq, sx, idx = activation_stages(L, X, tau, path)
        flag = oracle.detect_outliers(X, tau)
        Xq_o, sx_o = oracle.quantize_activations(X, flag)
        assert_equal(host(idx), oracle.compact(flag), f"idx tau={tau}")
        assert_equal(host(Xq), Xq_o, f"Xq tau={tau}")
        assert_equal(host(sx).view(np.uint32), sx_o.view(np.uint32), f"sx tau={tau}")
    ok_status(L)


@pytest.mark.parametrize("path", [1, 2])
def test_detect_edge_values(L, oracle, path):
    K = 64
    X = np.zeros((4, K), np.float16)
    X[0, 3] = 6.0                          # exactly the threshold: an outlier
    X[1, 5] = np.nextafter(np.float16(6.0), np.float16(0))  # just below: not
    X[2, 9] = -6.0
    X[2, 10] = 1.5
    X[3, :] = 0.0                          # zero row: scale 0, codes 0
    Xq, sx, idx = activation_stages(L, X, 6.0, path)
    assert host(idx).tolist() == [3, 9]
    flag = oracle.detect_outliers(X, 6.0)
    Xq_o, sx_o = oracle.quantize_activations(X, flag)
    assert_equal(host(Xq), Xq_o, "Xq")
    assert_equal(host(sx).view(np.uint32), sx_o.view(np.uint32), "sx")
    assert host(sx)[3] == 0.0


@pytest.mark.parametrize("path", [1, 2])
def test_detect_thresholds_between_halves(L, oracle, path):
    """Thresholds that are not fp16 values (between two halves, below the
    smallest subnormal, above the largest finite half, negative): the test
    |x| >= tau is the binary32 one."""
    pos = np.arange(0, 0x7c00, dtype=np.uint16)
    vals = np.concatenate([pos, pos | 0x8000]).view(np.float16)
    T = 16
    X = np.ascontiguousarray(vals[np.random.default_rng(3).permutation(vals.size)][: T * 3968].reshape(T, 3968))
    for tau in (6.0001, float(np.nextafter(np.float32(6.0), np.float32(0))), 1e-8, 70000.0, 65504.0, -1.0,
                0.0):
        flag = oracle.detect_outliers(X, tau)
        idx_o = oracle.compact(flag)
        Xq_o, sx_o = oracle.quantize_activations(X, flag)
        Xq, sx, idx = activation_stages(L, X, tau, path)
        assert_equal(host(idx), idx_o, f"idx tau={tau}")
        assert_equal(host(sx).view(np.uint32), sx_o.view(np.uint32), f"sx tau={tau}")
        assert_equal(host(Xq), Xq_o, f"Xq tau={tau}")
    ok_status(L)


@pytest.mark.parametrize("T,K", [(37, 1040), (520, 1040), (2100, 272), (129, 16)])
def test_detect_nonpositive_threshold_ragged(L, oracle, T, K):
    """tau <= 0 flags every column, and no more: K not a multiple of the
    detection strip, row counts that leave the strip's scanners partly idle
    (padding must never count as data)."""
    X, _ = synth.make_activations(T, K, seed=T + K, n_dims=2, mag=(6.0, 60.0))
    for tau in (0.0, -1.0):
        Xq, sx, idx = activation_stages(L, X, tau, 2)
        assert_equal(host(idx), np.arange(K, dtype=np.int32), f"idx tau={tau}")
        assert not host(Xq).any() and not host(sx).any()
    ok_status(L)


def every_fp16_rows(K, seed):
    """Every finite fp16 value (both zeros included) once, shuffled into rows
    of K, plus rows that put every value below a chosen row maximum under that
    maximum's scale (so small codes and every rounding boundary are reached)."""
    pos = np.arange(0, 0x7c00, dtype=np.uint16)
    vals = np.concatenate([pos, pos | 0x8000]).view(np.float16)
    rng = np.random.default_rng(seed)
    rows = [vals[rng.permutation(vals.size)][: (vals.size // K) * K].reshape(-1, K)]
    for amax in (np.float16(127 * 2.0 ** -7), np.float16(0.37), np.float16(1.0), np.float16(5.99),
                 np.float16(127.0), np.float16(3000.0)):
        below = vals[np.abs(vals.astype(np.float32)) <= np.float32(amax)]
        take = below[rng.permutation(below.size)][: (below.size // (K - 1)) * (K - 1)].reshape(-1, K - 1)
        take = take[:64]
        rows.append(np.concatenate([take, np.full((take.shape[0], 1), amax, np.float16)], axis=1))
    return np.ascontiguousarray(np.concatenate(rows))


@pytest.mark.parametrize("path", [1, 2])
def test_codes_every_fp16_value(L, oracle, path):
    """Each finite fp16 value as an activation and as a weight element, under
    many row scales, tau = inf (every column regular): the codes and scales
    agree bit for bit with the oracle's IEEE quotient, rounded half to even."""
    X = every_fp16_rows(256, seed=5 + path)
    rows = [X[i:i + 16] for i in range(0, X.shape[0], 16)] if path == 1 else [X]
    for Xr in rows:
        Xq, sx, _ = activation_stages(L, np.ascontiguousarray(Xr), float("inf"), path)
        Xq_o, sx_o = oracle.quantize_activations(Xr, np.zeros(Xr.shape[1], np.uint8))
        assert_equal(host(sx).view(np.uint32), sx_o.view(np.uint32), "sx")
        assert_equal(host(Xq), Xq_o, "Xq")
    Wq, sw = L.llmint8_quantize_weight(dev(X))
    Wq_o, sw_o = oracle.quantize_weight(X)
    torch.cuda.synchronize()
    assert_equal(host(sw).view(np.uint32), sw_o.view(np.uint32), "Wscale")
    assert_equal(host(Wq), Wq_o, "Wq")
    ok_status(L)


def near_tie_rows(rng, nrows, K):
    """Rows of fp16 values whose binary32 quotient x/s lies within 2^-12 of a
    half-integer (or on it), s = max|row| / 127: the band where a
    division-free code must defer to the IEEE division."""
    pos = np.arange(1, 0x7bff, dtype=np.uint16).view(np.float16)
    rows = []
    for r in range(nrows):
        amax = np.float16(127 * 2.0 ** -5) if r % 4 == 0 else np.float16(rng.uniform(0.5, 5.9))
        s = np.float32(np.float32(amax) / np.float32(127.0))
        xs = pos[pos.astype(np.float32) < np.float32(amax)]
        v = xs.astype(np.float32) / s
        f = v - np.floor(v)
        near = xs[np.abs(f - np.float32(0.5)) <= np.float32(2.0 ** -12)]
        assert near.size > 0
        row = rng.choice(near, K) * np.where(rng.random(K) < 0.5, -1, 1).astype(np.float16)
        row[rng.integers(0, K)] = amax
        rows.append(row.astype(np.float16))
    return np.stack(rows)


@pytest.mark.parametrize("path", [1, 2])
def test_near_tie_codes(L, oracle, path):
    rng = np.random.default_rng(77 + path)
    X = near_tie_rows(rng, 16 if path == 1 else 96, 1024)
    Xq, sx, idx = activation_stages(L, X, float("inf"), path)
    Xq_o, sx_o = oracle.quantize_activations(X, np.zeros(X.shape[1], np.uint8))
    assert_equal(host(sx).view(np.uint32), sx_o.view(np.uint32), "sx")
    assert_equal(host(Xq), Xq_o, "Xq near ties")
    Wq, sw = L.llmint8_quantize_weight(dev(X))
    Wq_o, sw_o = oracle.quantize_weight(X)
    assert_equal(host(Wq), Wq_o, "Wq near ties")


# --------------------------------------------------------------- the matmul

SMALL = [
    # (path, T, N, K)
    (1, 1, 128, 256), (1, 3, 300, 272), (1, 16, 1000, 1024), (1, 7, 129, 16), (1, 16, 256, 4096),
    (2, 1, 256, 256), (2, 17, 300, 272), (2, 129, 513, 1040), (2, 256, 256, 128),
    (2, 300, 1000, 1024), (2, 16, 256, 16),
]


@pytest.mark.parametrize("path,T,N,K", SMALL)
@pytest.mark.parametrize("tau", [6.0, float("inf"), 0.0])
def test_matmul_small(L, oracle, path, T, N, K, tau):
    X, W = synth.random_case(T, K, N, seed=T + N + K, n_dims=min(5, K), mag=(6.0, 50.0))
    run_full(L, oracle, X, W, tau, path)


@pytest.mark.parametrize("T,N,K", [(1, 1000, 128), (2, 300, 4096), (3, 11008, 2048), (4, 513, 4096)])
@pytest.mark.parametrize("tau", [6.0, 0.0, float("inf"), 30.0])
def test_decode_small_t_thresholds(L, oracle, T, N, K, tau):
    """Decode with T <= 4 and K % 128 == 0 (3-D weight copies): every
    intermediate (Xq, sx, the outlier list, int32 acc) bit-exact, Y within
    tolerance; tau = 0 makes every column an outlier (|O| = K), tau = inf none."""
    assert L.llmint8_kernel_launches(T, N, K) == 2
    X, W = synth.random_case(T, K, N, seed=T * 7 + K, n_dims=min(4, K), mag=(6.0, 50.0))
    run_full(L, oracle, X, W, tau, 1)


@pytest.mark.parametrize("T,N,K", [(3, 20011, 512), (16, 38000, 256), (1, 19000, 16)])
def test_decode_many_rows_per_cta(L, oracle, T, N, K):
    """N large enough that each GEMV CTA takes two or three chunks of rows
    (N / 148 > 128), with a ragged last slab; K both a multiple of 128 (3-D
    copies of several k-blocks) and not (2-D copies)."""
    X, W = synth.random_case(T, K, N, seed=T + N, n_dims=3, mag=(6.0, 40.0))
    run_full(L, oracle, X, W, 6.0, 1)


@pytest.mark.parametrize("path,T", [(1, 16), (1, 1), (2, 200)])
def test_maximum_k(L, oracle, path, T):
    """K = 65536, the largest K the library takes: the decode prep kernel's
    per-CTA slice is full (1024 chunks of 8 columns), the GEMV streams 128
    stages per row slab, the GEMM runs 512 k-blocks per tile."""
    assert L.llmint8_workspace_bytes(T, 300, 65536) > 0
    assert L.llmint8_workspace_bytes(T, 300, 65536 + 16) == 0
    X, W = synth.random_case(T, 65536, 300, seed=T + 65536, n_dims=6, mag=(6.0, 50.0))
    run_full(L, oracle, X, W, 6.0, path)


@pytest.mark.parametrize("path", [1, 2])
def test_tiny_config(L, oracle, path):
    w = synth.workload("tiny")
    run_full(L, oracle, w["X"], w["W"], 6.0, path)
    Xq, sx, idx = activation_stages(L, w["X"], 6.0, path)
    assert host(idx).tolist() == [7, 100]


def test_decode_7b_full(L, oracle):
    w = synth.workload("7b_decode")
    X16, W = w["X"], w["W"]
    Wq_o, sw_o = oracle.quantize_weight(W)
    Wd = dev(W)
    Wq, sw = L.llmint8_quantize_weight(Wd)
    assert_equal(host(Wq), Wq_o, "Wq")
    assert_equal(host(sw).view(np.uint32), sw_o.view(np.uint32), "Wscale")
    ws = L.alloc_workspace(16, W.shape[0], W.shape[1], "cuda")
    for T in (1, 2, 4, 8, 16):
        X = np.ascontiguousarray(X16[:T])
        Y_o, im = oracle.matmul(X, Wq_o, sw_o, W, 6.0, intermediates=True)
        Y, acc, Xq, sx, idx = L.llmint8_matmul_intermediates(dev(X), Wq, sw, Wd, 6.0, workspace=ws)
        Y2 = L.llmint8_matmul(dev(X), Wq, sw, Wd, 6.0, workspace=ws)
        torch.cuda.synchronize()
        assert im["nO"] == 4
        assert_equal(host(idx), im["idx"], f"idx T={T}")
        assert_equal(host(Xq), im["Xq"], f"Xq T={T}")
        assert_equal(host(sx).view(np.uint32), im["sx"].view(np.uint32), f"sx T={T}")
        assert_equal(host(acc), im["acc"], f"acc T={T}")
        assert_y_close(host(Y), Y_o, f"Y T={T}")
        assert_equal(host(Y2), host(Y), "debug and plain entry agree")
    ok_status(L)


def oracle_outlier_part(oracle, X, W, idx_o):
    """The oracle's fp part X[:, O] W[:, O]^T, computed on the gathered outlier
    columns: yo[t, n] = sum_j X[t, O_j] W[n, O_j] with the same terms in the
    same ascending order as on the full matrices (so the same binary64 sums),
    but reading contiguous rows, which keeps the full-size cases in seconds."""
    Xo = np.ascontiguousarray(X[:, idx_o])
    Wo = np.ascontiguousarray(W[:, idx_o])
    return oracle.outlier_gemm(Xo, Wo, np.arange(idx_o.size, dtype=np.int32))


def run_full_size(L, oracle, X, W, taus, seed=0):
    """Full-size check, every element: the integer stages (Wq, sw, the outlier
    list, Xq, sx) bit for bit, the int32 accumulator of all T x N outputs bit
    for bit against the oracle's int8 product (after a fast projection
    pre-check of every row), and every element of Y within the tolerance."""
    T, K = X.shape
    N = W.shape[0]
    Wq_o, sw_o = oracle.quantize_weight(W)
    Xd, Wd = dev(X), dev(W)
    Wq, sw = L.llmint8_quantize_weight(Wd)
    assert_equal(host(Wq), Wq_o, "Wq")
    assert_equal(host(sw).view(np.uint32), sw_o.view(np.uint32), "Wscale")
    ws = L.alloc_workspace(T, N, K, "cuda")
    acc = torch.empty((T, N), dtype=torch.int32, device="cuda")
    proj = projected_weights(Wq_o, seed=seed)
    for tau in taus:
        flag = oracle.detect_outliers(X, tau)
        idx_o = oracle.compact(flag)
        Xq_o, sx_o = oracle.quantize_activations(X, flag)
        Xq, sx, idx = L.llmint8_detect_quantize(Xd, tau)
        assert_equal(host(idx), idx_o, f"idx tau={tau}")
        assert_equal(host(Xq), Xq_o, f"Xq tau={tau}")
        assert_equal(host(sx).view(np.uint32), sx_o.view(np.uint32), f"sx tau={tau}")
        Y = L.llmint8_matmul_debug(Xd, Wq, sw, Wd, tau, workspace=ws, acc_out=acc)
        torch.cuda.synchronize()
        ok_status(L)
        acc_h = host(acc)
        assert_acc_exact(acc_h, Xq_o, proj, f"acc projections tau={tau}")
        acc_o = oracle.int8_gemm(Xq_o, Wq_o)
        assert_equal(acc_h, acc_o, f"acc every element tau={tau}")
        yo_o = oracle_outlier_part(oracle, X, W, idx_o) if idx_o.size else None
        Y_o = oracle.dequant_combine(acc_o, sx_o, sw_o, yo_o)
        del acc_o, yo_o
        assert_y_close(host(Y), Y_o, f"Y every element tau={tau}")
        del Y_o


def test_prefill_7b(L, oracle):
    w = synth.workload("7b_prefill")
    run_full_size(L, oracle, w["X"], w["W"], w["thresholds"], seed=1)


def test_upproj_13b(L, oracle):
    w = synth.workload("13b_up")
    run_full_size(L, oracle, w["X"], w["W"], w["thresholds"], seed=2)


def test_upproj_70b_threshold_sweep(L, oracle):
    w = synth.workload("70b_up")
    run_full_size(L, oracle, w["X"], w["W"], w["thresholds"], seed=3)


@pytest.mark.parametrize("tau", [6.0, 0.0, float("inf")])
def test_pair_gemm_many_tiles_per_pair(L, oracle, tau):
    """Every resident CTA pair of the persistent GEMM runs several tiles
    (T 600 = 3 row tiles, N 20000: hundreds of tiles for at most 74 pairs), so
    the hand-over between a pair's tiles (accumulator drain, weight-scale
    reload, outlier accumulator reset) is checked element by element."""
    X, W = synth.random_case(600, 1024, 20000, seed=600, n_dims=5, mag=(6.0, 50.0))
    run_full(L, oracle, X, W, tau, 2)


@pytest.mark.parametrize("tau", [6.0, 0.0])
def test_pair_gemm_ragged_edges(L, oracle, tau):
    """Many pair tiles per CTA pair with a ragged last row tile (T 520), N not
    a multiple of 8 (Y written with plain stores, a partial last tile) and K
    not a multiple of 128; tau 0 makes every column an outlier, so the fp16
    outlier products run over all of K; element by element."""
    X, W = synth.random_case(520, 1040, 20001, seed=520, n_dims=5, mag=(6.0, 50.0))
    run_full(L, oracle, X, W, tau, 2)


# --------------------------------------------------------------- int8 product alone

def saturated_codes(rng, T, K):
    """int8 codes over the full range, with rows of all +127, all -127, all
    -128 and alternating signs."""
    A = rng.integers(-128, 128, size=(T, K), dtype=np.int16).astype(np.int8)
    for r, v in enumerate((127, -127, -128)):
        if r < T:
            A[r] = v
    if T > 3:
        A[3] = np.where(np.arange(K) % 2 == 0, 127, -128).astype(np.int8)
    return A


@pytest.mark.parametrize("T,N,K", [(1, 300, 16), (5, 1001, 1040), (16, 4096, 4096), (17, 513, 272),
                                   (100, 300, 2048), (129, 777, 1024), (300, 1000, 4160),
                                   (600, 20000, 512)])
def test_int8_gemm_i32_bitexact(L, oracle, T, N, K):
    """acc = Xq Wq^T on arbitrary int8 codes (-128 included, saturated rows,
    adversarial signs), through each of the three kernels (GEMV T <= 16, one-CTA
    GEMM T <= 128, CTA-pair GEMM), with ragged T, N and K tails."""
    rng = np.random.default_rng(T * 1000 + N + K)
    Xq = saturated_codes(rng, T, K)
    Wq = saturated_codes(rng, N, K)
    acc = L.llmint8_int8_gemm_i32(dev(Xq), dev(Wq))
    torch.cuda.synchronize()
    ok_status(L)
    assert_equal(host(acc), oracle.int8_gemm(Xq, Wq), "acc")


@pytest.mark.parametrize("T", [3, 200])
def test_int8_gemm_i32_largest_k(L, oracle, T):
    """K = 65536 with every code at its extreme: |acc| reaches 65536 * 128^2 =
    2^30 (all -128 against all -128), the largest sum the entry allows."""
    K, N = 65536, 40
    rng = np.random.default_rng(T)
    Xq = saturated_codes(rng, T, K)
    Wq = saturated_codes(rng, N, K)
    acc = L.llmint8_int8_gemm_i32(dev(Xq), dev(Wq))
    torch.cuda.synchronize()
    ok_status(L)
    acc_o = oracle.int8_gemm(Xq, Wq)
    assert acc_o[2, 2] == 2 ** 30
    assert_equal(host(acc), acc_o, "acc")


def test_int8_gemm_i32_matches_the_matmul_accumulator(L, oracle):
    """The codes llmint8_matmul forms, multiplied by the standalone entry, give
    the accumulator the matmul itself reports."""
    X, W = synth.random_case(300, 1024, 640, seed=31, n_dims=4)
    Wd = dev(W)
    Wq, sw = L.llmint8_quantize_weight(Wd)
    _, acc, Xq, _, _ = L.llmint8_matmul_intermediates(dev(X), Wq, sw, Wd, 6.0)
    acc2 = L.llmint8_int8_gemm_i32(Xq, Wq)
    torch.cuda.synchronize()
    assert_equal(host(acc2), host(acc), "int8 product alone vs inside the matmul")


# --------------------------------------------------------------- robustness

def test_workspace_reuse_and_garbage(L, oracle):
    X, W = synth.random_case(300, 1040, 513, seed=5, n_dims=4)
    Wq_o, sw_o = oracle.quantize_weight(W)
    Wd = dev(W)
    Wq, sw = L.llmint8_quantize_weight(Wd)
    for path in (1, 2):
        nbytes = max(L.llmint8_workspace_bytes(300, 513, 1040, 2),
                     L.llmint8_workspace_bytes(16, 513, 1040, 1))
        ws = torch.randint(0, 255, (nbytes,), dtype=torch.uint8, device="cuda")
        for T in (16, 3, 300, 1, 16) if path == 2 else (16, 3, 1, 16):
            Xt = np.ascontiguousarray(X[:T])
            Y = L.llmint8_matmul_debug(dev(Xt), Wq, sw, Wd, 6.0, workspace=ws, path=path)
            Y_o = oracle.matmul(Xt, Wq_o, sw_o, W, 6.0)
            torch.cuda.synchronize()
            assert_y_close(host(Y), Y_o, f"path {path} T={T}")
    ok_status(L)


@pytest.mark.parametrize("path,T", [(1, 9), (2, 9), (2, 200)])
def test_output_guard_bands(L, oracle, path, T):
    N, K = 300, 272
    X, W = synth.random_case(T, K, N, seed=8)
    Wd = dev(W)
    Wq, sw = L.llmint8_quantize_weight(Wd)
    pad = 4096
    buf = torch.full((T * N + 2 * pad,), 1234.0, dtype=torch.float16, device="cuda")
    Y = buf[pad:pad + T * N].view(T, N)
    L.llmint8_matmul_debug(dev(X), Wq, sw, Wd, 6.0, Y=Y, path=path)
    torch.cuda.synchronize()
    assert bool((buf[:pad] == 1234.0).all()) and bool((buf[pad + T * N:] == 1234.0).all())
    assert_y_close(host(Y), oracle.matmul(X, *oracle.quantize_weight(W), W, 6.0), "Y")


def test_timeout_path_reports_and_recovers(L, oracle):
    assert L.llmint8_sync_status() == 0
    L.llmint8_selftest_timeout(2_000_000)  # 2 ms: nothing ever arrives on the barrier
    assert L.llmint8_sync_status() == L.llmint8.LLMINT8_ERR_TIMEOUT
    assert L.llmint8_sync_status() == 0    # cleared
    X, W = synth.random_case(16, 256, 256, seed=9)
    run_full(L, oracle, X, W, 6.0, 1)


def test_misaligned_pointer_rejected(L):
    X = torch.zeros((4, 64 + 8), dtype=torch.float16, device="cuda")
    W = torch.zeros((8, 64), dtype=torch.float16, device="cuda")
    Wq, sw = L.llmint8_quantize_weight(W)
    Xbad = X.view(-1)[1:1 + 4 * 64].view(4, 64)  # 2-byte offset
    ws = L.alloc_workspace(4, 8, 64, "cuda")
    with pytest.raises(L.LLMInt8Error) as e:
        L.llmint8_matmul(Xbad, Wq, sw, W, 6.0, workspace=ws)
    assert e.value.status == -2
    with pytest.raises(L.LLMInt8Error) as e:
        L.llmint8_matmul(X[:, :64].contiguous(), Wq, sw, W, float("nan"), workspace=ws)
    assert e.value.status == -1


def test_int8_linear_wrapper(L, oracle):
    X, W = synth.random_case(40, 512, 96, seed=10)
    lin = L.Int8Linear(dev(W))
    Y = lin(dev(X))
    Y1 = lin(dev(np.ascontiguousarray(X[:1])))
    torch.cuda.synchronize()
    Wq_o, sw_o = oracle.quantize_weight(W)
    assert_y_close(host(Y), oracle.matmul(X, Wq_o, sw_o, W, 6.0), "Y")
    assert_y_close(host(Y1), oracle.matmul(np.ascontiguousarray(X[:1]), Wq_o, sw_o, W, 6.0), "Y1")


@pytest.mark.parametrize("path", [1, 2])
def test_cuda_graph_replay_matches_direct_calls(L, oracle, path):
    """The calls chain with programmatic dependent launch; captured into a CUDA
    graph (as the benchmark and a decode loop run them) and replayed, they give
    the same bytes as direct calls."""
    T = 16 if path == 1 else 200
    X, W = synth.random_case(T, 1024, 640, seed=40 + path, n_dims=3)
    X2, _ = synth.random_case(T, 1024, 640, seed=50 + path, n_dims=5)
    Wd = dev(W)
    Wq, sw = L.llmint8_quantize_weight(Wd)
    ws = L.alloc_workspace(T, 640, 1024, "cuda", path)
    Xd, X2d = dev(X), dev(X2)
    Y1 = torch.empty((T, 640), dtype=torch.float16, device="cuda")
    Y2 = torch.empty_like(Y1)
    L.llmint8_matmul_debug(Xd, Wq, sw, Wd, 6.0, workspace=ws, Y=Y1, path=path)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        L.llmint8_matmul_debug(Xd, Wq, sw, Wd, 6.0, workspace=ws, Y=Y1, path=path)
        L.llmint8_matmul_debug(X2d, Wq, sw, Wd, 6.0, workspace=ws, Y=Y2, path=path)
    Y1.zero_()
    Y2.zero_()
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    ok_status(L)
    Wq_o, sw_o = oracle.quantize_weight(W)
    assert_y_close(host(Y1), oracle.matmul(X, Wq_o, sw_o, W, 6.0), "graph Y1")
    assert_y_close(host(Y2), oracle.matmul(X2, Wq_o, sw_o, W, 6.0), "graph Y2")
    Yd = L.llmint8_matmul_debug(X2d, Wq, sw, Wd, 6.0, workspace=ws, path=path)
    torch.cuda.synchronize()
    assert_equal(host(Yd), host(Y2), "graph replay and direct call agree")


@pytest.mark.parametrize("path", [1, 2])
def test_profile_repeats_recompute_same_y(L, oracle, path):
    """The profiling entry relaunches the main kernel on one workspace; every
    launch must recompute the same Y."""
    T = 7 if path == 1 else 150
    X, W = synth.random_case(T, 2048, 700, seed=60 + path, n_dims=4)
    Wd = dev(W)
    Wq, sw = L.llmint8_quantize_weight(Wd)
    ws = L.alloc_workspace(T, 700, 2048, "cuda", path)
    Y0 = L.llmint8_matmul_debug(dev(X), Wq, sw, Wd, 6.0, workspace=ws, path=path)
    Y1 = torch.zeros_like(Y0)
    b = torch.cuda.Event(enable_timing=True)
    e = torch.cuda.Event(enable_timing=True)
    L.llmint8_matmul_profile(dev(X), Wq, sw, Wd, 6.0, ws, Y1, b, e, repeat=5, path=path)
    torch.cuda.synchronize()
    ok_status(L)
    assert b.elapsed_time(e) > 0
    assert_equal(host(Y1), host(Y0), "profile repeats")
    Wq_o, sw_o = oracle.quantize_weight(W)
    assert_y_close(host(Y1), oracle.matmul(X, Wq_o, sw_o, W, 6.0), "Y")


@pytest.mark.parametrize("path", [1, 2])
def test_weight_rewritten_just_before_a_call_is_seen(L, oracle, path):
    """The kernels request Wq before the kernel queued ahead of them is done
    (programmatic dependent launch).  A weight quantised into the same Wq
    buffer right before a call, on the same stream, must still be the one the
    call reads: the weight kernel does not let its dependents start early."""
    T = 16 if path == 1 else 300
    N, K = 1500, 2048
    X, W1 = synth.random_case(T, K, N, seed=70 + path, n_dims=4)
    W2 = synth.make_weight(N, K, seed=80 + path, sigma=0.07)
    W1d, W2d, Xd = dev(W1), dev(W2), dev(X)
    Wq, sw = L.llmint8_quantize_weight(W1d)
    ws = L.alloc_workspace(T, N, K, "cuda", path)
    Y1 = L.llmint8_matmul_debug(Xd, Wq, sw, W1d, 6.0, workspace=ws, path=path)
    L.llmint8_quantize_weight(W2d, Wq, sw)          # overwrite in place, same stream
    Y2 = L.llmint8_matmul_debug(Xd, Wq, sw, W2d, 6.0, workspace=ws, path=path)
    Wq.copy_(torch.zeros_like(Wq))                   # a torch kernel writes Wq, then a call
    Y3 = L.llmint8_matmul_debug(Xd, Wq, sw, W2d, 6.0, workspace=ws, path=path)
    torch.cuda.synchronize()
    ok_status(L)
    Wq1, sw1 = oracle.quantize_weight(W1)
    Wq2, sw2 = oracle.quantize_weight(W2)
    assert_y_close(host(Y1), oracle.matmul(X, Wq1, sw1, W1, 6.0), "first weight")
    assert_y_close(host(Y2), oracle.matmul(X, Wq2, sw2, W2, 6.0), "rewritten weight")
    assert_y_close(host(Y3), oracle.matmul(X, np.zeros_like(Wq2), sw2, W2, 6.0), "zeroed codes")
