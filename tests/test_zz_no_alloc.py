"""The allocation-free decode entry point (collected last on purpose).

llmint8_matmul_decode_noalloc serves callers that cannot allocate device
memory, such as a host program whose allocator owns every byte of the device
or a decode loop where an allocation could stall or fail mid-run: its scratch
is one fixed array per GPU inside the library.  It runs the same kernels as
the workspace entry point llmint8_matmul, so on the same inputs the two must
give the same bytes; both are also checked against the CPU oracle within the
tolerance of the other parity tests.  Two calls in a row per shape: the second
shows that what the first left in the shared array does no harm.
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


# (N, K, the T of two calls in a row): K % 128 == 0 (3-D weight copies), K not a
# multiple of 128 (2-D copies), and the largest K the scratch array takes.
SHAPES = [(3000, 4096, (16, 3)), (1000, 1040, (5, 16)), (700, 16384, (16, 1))]


@pytest.mark.parametrize("N,K,Ts", SHAPES)
def test_noalloc_matches_workspace_entry_and_oracle(L, oracle, N, K, Ts):
    Wh = synth.make_weight(N, K, seed=91 + K)
    W = torch.from_numpy(Wh).cuda()
    Wq, sw = L.llmint8_quantize_weight(W)
    Wq_o, sw_o = oracle.quantize_weight(Wh)
    ws = L.alloc_workspace(16, N, K, "cuda")
    for call, T in enumerate(Ts):
        Xh, _ = synth.make_activations(T, K, seed=92 + call + K, n_dims=4, mag=(6.0, 60.0))
        X = torch.from_numpy(Xh).cuda()
        Y_ref = L.llmint8_matmul(X, Wq, sw, W, 6.0, workspace=ws)
        Y = L.llmint8_matmul_decode_noalloc(X, Wq, sw, W, 6.0)
        torch.cuda.synchronize()
        assert L.llmint8_sync_status() == 0
        assert_equal(Y.cpu().numpy().view(np.uint16), Y_ref.cpu().numpy().view(np.uint16),
                     f"call {call}: no-alloc and workspace entries")
        Y_o = oracle.matmul(Xh, Wq_o, sw_o, Wh, 6.0)
        assert_y_close(Y.cpu().numpy(), Y_o, f"call {call} T={T}: no-alloc entry vs oracle")


def test_noalloc_rejects_sizes_past_its_limits(L):
    W = torch.zeros((8, 64), dtype=torch.float16, device="cuda")
    Wq, sw = L.llmint8_quantize_weight(W)
    with pytest.raises(L.LLMInt8Error) as e:
        L.llmint8_matmul_decode_noalloc(torch.zeros((17, 64), dtype=torch.float16, device="cuda"),
                                        Wq, sw, W)
    assert e.value.status == -1
    Wbig = torch.zeros((8, 16400), dtype=torch.float16, device="cuda")
    Wqb, swb = L.llmint8_quantize_weight(Wbig)
    with pytest.raises(L.LLMInt8Error) as e:
        L.llmint8_matmul_decode_noalloc(torch.zeros((2, 16400), dtype=torch.float16, device="cuda"),
                                        Wqb, swb, Wbig)
    assert e.value.status == -1


def test_noalloc_binding_rejects_mismatched_shapes(L):
    """The C entry point sees only pointers; the binding refuses buffers that
    are shorter than the sizes imply before anything is launched."""
    X = torch.zeros((4, 64), dtype=torch.float16, device="cuda")
    W = torch.zeros((8, 64), dtype=torch.float16, device="cuda")
    Wq, sw = L.llmint8_quantize_weight(W)
    with pytest.raises(ValueError):
        L.llmint8_matmul_decode_noalloc(X, Wq, sw, W[:, :48].contiguous())
    with pytest.raises(ValueError):
        L.llmint8_matmul_decode_noalloc(X, Wq, sw[:4].contiguous(), W)
    with pytest.raises(ValueError):
        L.llmint8_matmul_decode_noalloc(X, Wq, sw, W,
                                        Y=torch.empty((4, 7), dtype=torch.float16, device="cuda"))
