"""The C-ABI library without a GPU: it builds, loads, exports every entry point
include/llmint8.h declares, and rejects bad arguments before any CUDA call.

Only host-side paths run here: argument validation returns before the library
touches the device, so fake (never dereferenced) pointers are safe.
"""
import ctypes
import os
import re
import subprocess

import pytest

import int8_mixed_precision_outlier_b200 as L
from int8_mixed_precision_outlier_b200 import _build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    _build.build()
    return L.load_library()


def test_every_declared_symbol_is_exported(lib):
    names = L.header_functions()
    assert len(names) >= 10
    for n in names:
        assert getattr(lib, n) is not None
    out = subprocess.run(["nm", "-D", "--defined-only", _build.LIB], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\sT\s(llmint8_\w+)", out))
    assert exported == set(names)


def test_status_strings_and_version(lib):
    assert L.llmint8_version() >= 100
    for s in range(-7, 1):
        assert L.llmint8_status_string(s)
    assert "timeout" in L.llmint8_status_string(-6) or "bounded wait" in L.llmint8_status_string(-6)


def test_workspace_sizes(lib):
    ws = L.llmint8_workspace_bytes
    assert ws(16, 11008, 4096) == ws(16, 11008, 4096, L.PATH_GEMV)
    assert ws(17, 11008, 4096) == ws(17, 11008, 4096, L.PATH_GEMM)
    assert ws(17, 11008, 4096, L.PATH_GEMV) == 0          # decode path takes T <= 16 only
    assert ws(4, 100, 24) == 0 and ws(4, 100, 8) == 0      # K must be a multiple of 16, >= 16
    assert ws(4, 100, 65536 + 16) == 0                     # K limit
    # the prefill workspace holds Xq, the gathered Xo and Wo at worst case |O| = K
    T, N, K = 2048, 4096, 4096
    assert ws(T, N, K) >= T * K + 2 * T * K + 2 * N * K
    assert ws(T, 2 * N, K) > ws(T, N, K)


def test_kernel_launch_counts(lib):
    kl = L.llmint8_kernel_launches
    assert kl(1, 11008, 4096) == 2 and kl(16, 11008, 4096) == 2     # prep kernel + GEMV
    assert kl(4, 11008, 4160) == 2 and kl(2, 100, 8192) == 2
    assert kl(17, 4096, 4096) == 3 and kl(2048, 4096, 4096) == 3     # detect, quantize + gathers, GEMM
    assert kl(4, 100, 256, L.PATH_GEMM) == 3
    assert kl(0, 100, 256) == 0 and kl(4, 0, 256) == 0 and kl(4, 100, 24) == 0


def _fake(addr):
    return ctypes.c_void_p(addr)


def test_validation_before_any_device_call(lib):
    A = _fake(0x10000)  # aligned, never dereferenced: validation fails first
    big = 1 << 40
    # NaN threshold
    assert lib.llmint8_matmul(A, 4, 64, A, A, A, 8, float("nan"), A, A, big, None) == -1
    # K not a multiple of 16
    assert lib.llmint8_matmul(A, 4, 72, A, A, A, 8, 6.0, A, A, big, None) == -2
    # misaligned X
    assert lib.llmint8_matmul(_fake(0x10002), 4, 64, A, A, A, 8, 6.0, A, A, big, None) == -2
    # workspace too small
    assert lib.llmint8_matmul(A, 4, 64, A, A, A, 8, 6.0, A, A, 16, None) == -4
    # null workspace / null output
    assert lib.llmint8_matmul(A, 4, 64, A, A, A, 8, 6.0, A, None, big, None) == -1
    assert lib.llmint8_matmul(A, 4, 64, A, A, A, 8, 6.0, None, A, big, None) == -1
    # bad path; decode path with T > 16
    nil = (None, None, None, None, None)
    assert lib.llmint8_matmul_debug(A, 4, 64, A, A, A, 8, 6.0, A, A, big, 7, *nil, None) == -1
    assert lib.llmint8_matmul_debug(A, 17, 64, A, A, A, 8, 6.0, A, A, big, 1, *nil, None) == -1
    # misaligned inspection output
    assert lib.llmint8_matmul_debug(A, 4, 64, A, A, A, 8, 6.0, A, A, big, 1, None, _fake(0x10001),
                                    None, None, None, None) == -2
    # activation stages alone: the decode path takes T <= 16 only
    assert lib.llmint8_detect_quantize(A, 17, 64, 6.0, A, A, A, A, A, big, 1, None) == -1
    # K so large that an int32 sum could overflow
    assert lib.llmint8_matmul(A, 4, 140000, A, A, A, 8, 6.0, A, A, big, None) == -1
    # weight quantisation
    assert lib.llmint8_quantize_weight(A, 8, 8, A, A, None) == -1
    assert lib.llmint8_quantize_weight(A, 8, 24, A, A, None) == -2
    assert lib.llmint8_quantize_weight(None, 8, 64, A, A, None) == -1
    # empty problems are valid no-ops
    assert lib.llmint8_matmul(None, 0, 64, A, A, A, 8, 6.0, A, None, 0, None) == 0
    assert lib.llmint8_matmul(A, 4, 64, A, A, A, 0, 6.0, A, A, big, None) == 0
    assert lib.llmint8_quantize_weight(A, 0, 64, A, A, None) == 0
    # wait limit bounds
    assert lib.llmint8_set_wait_limit_ns(10) == -1
    assert lib.llmint8_set_wait_limit_ns(2_000_000_000) == 0
    assert lib.llmint8_selftest_timeout(10, None) == -1


def test_noalloc_limits_checked_before_any_device_call(lib):
    A = _fake(0x10000)
    f = lib.llmint8_matmul_decode_noalloc
    assert f(A, 17, 64, A, A, A, 8, 6.0, A, None) == -1        # T > 16: not a decode shape
    assert f(A, 4, 16384 + 16, A, A, A, 8, 6.0, A, None) == -1  # K past the scratch limit
    assert f(A, 4, 64, A, A, A, 1 << 31, 6.0, A, None) == -1      # N past int32
    assert f(A, 4, 72, A, A, A, 8, 6.0, A, None) == -1          # K % 16 != 0
    assert f(A, -1, 64, A, A, A, 8, 6.0, A, None) == -1
    assert f(None, 0, 64, A, A, A, 8, 6.0, A, None) == 0        # empty problems are no-ops
    assert f(A, 4, 64, A, A, A, 0, 6.0, A, None) == 0


def test_missing_library_fails_loudly(tmp_path):
    from int8_mixed_precision_outlier_b200 import llmint8 as B
    with pytest.raises(OSError):
        B._declare  # noqa: B018  (module loads fine without the library)
        saved = B._LIB
        try:
            B._LIB = None
            B.load_library(str(tmp_path / "nope.so"))
        finally:
            B._LIB = saved


def test_product_code_never_touches_the_oracle():
    pkg = os.path.join(ROOT, "int8_mixed_precision_outlier_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                src = open(os.path.join(dirpath, f), encoding="utf-8").read()
                assert not re.search(r"^\s*(from|import)\s+oracle", src, re.M), f
                assert "llmint8_oracle" not in src, f
                assert "liboracle" not in src, f


def test_binding_shape_checks_run_before_any_launch():
    """check_matmul_shapes (run by every matmul wrapper before its C call)
    refuses any buffer whose shape disagrees with X [T, K] and Wq [N, K]: the
    C side sees only pointers and would read or write past the end."""
    import torch
    T, N, K = 4, 8, 64
    X = torch.zeros((T, K), dtype=torch.float16)
    Wq = torch.zeros((N, K), dtype=torch.int8)
    sw = torch.zeros(N, dtype=torch.float32)
    W = torch.zeros((N, K), dtype=torch.float16)
    Y = torch.zeros((T, N), dtype=torch.float16)
    L.check_matmul_shapes(X, Wq, sw, W, Y)            # consistent: no error
    L.check_matmul_shapes(X, Wq, sw, None, Y)         # W optional
    bad = [dict(W=torch.zeros((N, K - 16), dtype=torch.float16)),
           dict(W=torch.zeros((N + 1, K), dtype=torch.float16)),
           dict(Wscale=torch.zeros(N - 1, dtype=torch.float32)),
           dict(Wq=torch.zeros((N, K - 16), dtype=torch.int8)),
           dict(Y=torch.zeros((T, N - 1), dtype=torch.float16)),
           dict(Y=torch.zeros((T + 1, N), dtype=torch.float16)),
           dict(acc_out=torch.zeros((T, N - 1), dtype=torch.int32)),
           dict(xq_out=torch.zeros((T, K - 16), dtype=torch.int8)),
           dict(sx_out=torch.zeros(T - 1, dtype=torch.float32)),
           dict(idx_out=torch.zeros(K - 1, dtype=torch.int32))]
    for b in bad:
        args = dict(X=X, Wq=Wq, Wscale=sw, W=W, Y=Y)
        args.update(b)
        with pytest.raises(ValueError):
            L.check_matmul_shapes(**args)


def test_int8_gemm_i32_validation_before_any_device_call(lib):
    A = _fake(0x10000)
    f = lib.llmint8_int8_gemm_i32
    assert f(A, A, 4, 8, 72, A, None) == -2               # K % 16 != 0
    assert f(A, A, 4, 8, 8, A, None) == -1                # K < 16
    assert f(A, A, 4, 8, 65536 + 16, A, None) == -1       # K past the limit
    assert f(_fake(0x10008), A, 4, 8, 64, A, None) == -2  # misaligned Xq
    assert f(A, A, 4, 8, 64, _fake(0x10002), None) == -2  # misaligned acc
    assert f(None, A, 4, 8, 64, A, None) == -1
    assert f(A, A, -1, 8, 64, A, None) == -1
    assert f(None, None, 0, 8, 64, None, None) == 0       # empty problems are no-ops
    assert f(A, A, 4, 0, 64, A, None) == 0


def test_smoothquant_validation_before_any_device_call(lib):
    A = _fake(0x10000)
    big = 1 << 40
    assert lib.llmint8_smooth_factors(A, A, 64, 1.5, A, None) == -1           # alpha outside [0, 1]
    assert lib.llmint8_smooth_factors(A, A, 64, float("nan"), A, None) == -1
    assert lib.llmint8_smooth_factors(A, A, 0, 0.5, A, None) == 0             # empty
    assert lib.llmint8_column_absmax(A, 4, 72, A, 0, None) == -2              # K % 16
    assert lib.llmint8_column_absmax(_fake(0x10008), 4, 64, A, 0, None) == -2
    assert lib.llmint8_smoothquant_quantize_weight(A, 8, 64, _fake(0x10004), A, A, None) == -2  # s misaligned
    assert lib.llmint8_smoothquant_workspace_bytes(4, 72) == 0
    assert lib.llmint8_smoothquant_workspace_bytes(2048, 4096) >= 2048 * 4096 + 4 * 2048
    f = lib.llmint8_smoothquant_matmul
    assert f(A, 4, 64, A, A, A, 8, A, A, 16, None) == -4                      # workspace too small
    assert f(A, 4, 64, None, A, A, 8, A, A, big, None) == -1                  # no factors
    assert f(A, 4, 64, A, A, A, 0, A, A, big, None) == 0                      # empty
    d = lib.llmint8_smoothquant_matmul_debug
    assert d(A, 17, 64, A, A, A, 8, A, A, big, 1, None, None, None, None) == -1  # GEMV path, T > 16
