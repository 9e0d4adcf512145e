"""The allocation-free decode entry point (collected last on purpose).

llmint8_matmul_decode_noalloc serves callers that cannot allocate device
memory: its scratch is one fixed array per GPU inside the library.  Two calls
in a row must each match the workspace entry point llmint8_matmul on the same
inputs, within the tolerance of the other parity tests -- the second call also
shows that what the first left in the shared array does no harm.
"""
import numpy as np
import pytest

from gpu_helpers import assert_y_close
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


def test_noalloc_matches_workspace_entry_two_calls_in_a_row(L):
    N, K = 3000, 4096
    W = torch.from_numpy(synth.make_weight(N, K, seed=91)).cuda()
    Wq, sw = L.llmint8_quantize_weight(W)
    ws = L.alloc_workspace(16, N, K, "cuda")
    for call, (T, seed) in enumerate(((16, 92), (3, 93))):
        X = torch.from_numpy(synth.make_activations(T, K, seed=seed, n_dims=4)[0]).cuda()
        Y_ref = L.llmint8_matmul(X, Wq, sw, W, 6.0, workspace=ws)
        Y = L.llmint8_matmul_decode_noalloc(X, Wq, sw, W, 6.0)
        torch.cuda.synchronize()
        assert L.llmint8_sync_status() == 0
        assert_y_close(Y.cpu().numpy(), Y_ref.cpu().numpy(), f"call {call}")


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
