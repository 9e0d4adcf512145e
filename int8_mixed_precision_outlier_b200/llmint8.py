"""Python binding of the C ABI in include/llmint8.h.

Argument marshalling only: every function takes torch CUDA tensors, checks
dtypes and shapes, and passes raw device pointers, sizes and the current CUDA
stream to `libllmint8.so`.  Every step of the computation runs in the
library's sm_100a kernels.  There is no CPU or PyTorch fallback: if the
library cannot be loaded, the calls raise.
"""
from __future__ import annotations

import ctypes
import os
import re
import threading

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libllmint8.so")
HEADER = os.path.join(os.path.dirname(_PKG), "include", "llmint8.h")

LLMINT8_OK = 0
LLMINT8_ERR_INVALID_ARG = -1
LLMINT8_ERR_TIMEOUT = -6
PATH_AUTO, PATH_GEMV, PATH_GEMM = 0, 1, 2
GEMV_MAX_T = 16

_LOCK = threading.Lock()
_LIB = None


class LLMInt8Error(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {llmint8_status_string(status)} (status {status})")


def _declare(lib):
    P, I64, F, I, SZ, U64 = (ctypes.c_void_p, ctypes.c_int64, ctypes.c_float, ctypes.c_int,
                             ctypes.c_size_t, ctypes.c_uint64)
    sig = {
        "llmint8_status_string": (ctypes.c_char_p, [I]),
        "llmint8_version": (I, []),
        "llmint8_quantize_weight": (I, [P, I64, I64, P, P, P]),
        "llmint8_workspace_bytes": (SZ, [I64, I64, I64]),
        "llmint8_workspace_bytes_path": (SZ, [I64, I64, I64, I]),
        "llmint8_kernel_launches": (I, [I64, I64, I64, I]),
        "llmint8_matmul": (I, [P, I64, I64, P, P, P, I64, F, P, P, SZ, P]),
        "llmint8_matmul_debug": (I, [P, I64, I64, P, P, P, I64, F, P, P, SZ, I, P, P, P, P, P, P]),
        "llmint8_matmul_profile": (I, [P, I64, I64, P, P, P, I64, F, P, P, SZ, I, I, P, P, P]),
        "llmint8_detect_quantize": (I, [P, I64, I64, F, P, P, P, P, P, SZ, I, P]),
        "llmint8_matmul_decode_noalloc": (I, [P, I64, I64, P, P, P, I64, F, P, P]),
        "llmint8_int8_gemm_i32": (I, [P, P, I64, I64, I64, P, P]),
        "llmint8_outlier_store_build": (I, [P, I64, I64, P, I64, P, P, P]),
        "llmint8_matmul_stored": (I, [P, I64, I64, P, P, P, P, I64, F, P, P, P, SZ, P]),
        "llmint8_matmul_stored_debug": (I, [P, I64, I64, P, P, P, P, I64, F, P, P, P, SZ, I, P, P]),
        "llmint8_fp8_quantize_weight": (I, [P, I64, I64, P, P, P]),
        "llmint8_fp8_matmul": (I, [P, I64, I64, P, P, P, I64, F, P, P, SZ, P]),
        "llmint8_fp8_matmul_debug": (I, [P, I64, I64, P, P, P, I64, F, P, P, SZ, I, P, P, P, P, P, P]),
        "llmint8_column_absmax": (I, [P, I64, I64, P, I, P]),
        "llmint8_smooth_factors": (I, [P, P, I64, F, P, P]),
        "llmint8_smoothquant_quantize_weight": (I, [P, I64, I64, P, P, P, P]),
        "llmint8_smoothquant_workspace_bytes": (SZ, [I64, I64]),
        "llmint8_smoothquant_matmul": (I, [P, I64, I64, P, P, P, I64, P, P, SZ, P]),
        "llmint8_smoothquant_matmul_debug": (I, [P, I64, I64, P, P, P, I64, P, P, SZ, I, P, P, P, P]),
        "llmint8_sync_status": (I, [P]),
        "llmint8_selftest_timeout": (I, [U64, P]),
        "llmint8_set_wait_limit_ns": (I, [U64]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


def load_library(path: str | None = None):
    """Load (once) and return the ctypes handle of libllmint8.so."""
    global _LIB
    with _LOCK:
        if _LIB is None:
            p = path or LIB_PATH
            if not os.path.exists(p):
                raise OSError(f"{p} is missing: build it with __graft_entry__.build() or "
                              "python -m int8_mixed_precision_outlier_b200._build")
            _LIB = _declare(ctypes.CDLL(p))
        return _LIB


def header_functions() -> list[str]:
    """Names of the entry points include/llmint8.h declares."""
    with open(HEADER, encoding="utf-8") as f:
        src = f.read()
    return sorted(set(re.findall(r"LLMINT8_API\s+[\w\s\*]*?\b(llmint8_\w+)\s*\(", src)))


def _check(status: int, where: str):
    if status != LLMINT8_OK:
        raise LLMInt8Error(status, where)


def _ptr(t: torch.Tensor | None):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _need(t: torch.Tensor, dtype, ndim: int, name: str):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if t.dim() != ndim or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous {ndim}-D tensor")


def check_matmul_shapes(X, Wq, Wscale, W, Y=None, acc_out=None, xq_out=None, sx_out=None,
                        idx_out=None, n_out=None):
    """Shape and device agreement of a matmul's tensors (dtypes are checked
    separately).  The C entry points only see pointers, so a buffer shorter
    than the sizes imply would be read or written past its end on the device:
    every mismatch raises ValueError here, before any launch.  W may be None
    (calls that do not read the fp16 weight)."""
    if X.dim() != 2 or Wq.dim() != 2:
        raise ValueError("X and Wq must be 2-D")
    T, K = X.shape
    N = Wq.shape[0]
    want = {"Wq": (Wq, (N, K)), "Wscale": (Wscale, (N,)), "W": (W, (N, K)), "Y": (Y, (T, N)),
            "acc_out": (acc_out, (T, N)), "xq_out": (xq_out, (T, K)), "sx_out": (sx_out, (T,)),
            "idx_out": (idx_out, (K,)), "n_out": (n_out, (1,))}
    for name, (t, shape) in want.items():
        if t is None:
            continue
        if tuple(t.shape) != shape:
            raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {shape} "
                             f"for X [{T}, {K}] and Wq [{N}, {K}]")
        if t.device != X.device:
            raise ValueError(f"{name} is on {t.device}, X on {X.device}")


# ------------------------------------------------------------------ host-only

def llmint8_status_string(status: int) -> str:
    return load_library().llmint8_status_string(int(status)).decode()


def llmint8_version() -> int:
    return int(load_library().llmint8_version())


def llmint8_workspace_bytes(T: int, N: int, K: int, path: int = PATH_AUTO) -> int:
    lib = load_library()
    if path == PATH_AUTO:
        return int(lib.llmint8_workspace_bytes(T, N, K))
    return int(lib.llmint8_workspace_bytes_path(T, N, K, path))


def llmint8_kernel_launches(T: int, N: int, K: int, path: int = PATH_AUTO) -> int:
    """Kernels one llmint8_matmul call of this shape launches (0 if rejected)."""
    return int(load_library().llmint8_kernel_launches(T, N, K, path))


def llmint8_set_wait_limit_ns(ns: int):
    _check(load_library().llmint8_set_wait_limit_ns(int(ns)), "llmint8_set_wait_limit_ns")


# ------------------------------------------------------------------ device calls

def llmint8_quantize_weight(W: torch.Tensor, Wq: torch.Tensor | None = None,
                            Wscale: torch.Tensor | None = None, stream=None):
    """W fp16 [N,K] -> (Wq int8 [N,K], Wscale fp32 [N])."""
    _need(W, torch.float16, 2, "W")
    N, K = W.shape
    Wq = torch.empty((N, K), dtype=torch.int8, device=W.device) if Wq is None else Wq
    Wscale = torch.empty(N, dtype=torch.float32, device=W.device) if Wscale is None else Wscale
    _need(Wq, torch.int8, 2, "Wq")
    _need(Wscale, torch.float32, 1, "Wscale")
    if tuple(Wq.shape) != (N, K) or tuple(Wscale.shape) != (N,) or Wq.device != W.device \
            or Wscale.device != W.device:
        raise ValueError(f"Wq must be [{N}, {K}] and Wscale [{N}] on {W.device}")
    _check(load_library().llmint8_quantize_weight(_ptr(W), N, K, _ptr(Wq), _ptr(Wscale),
                                                  _stream(stream)), "llmint8_quantize_weight")
    return Wq, Wscale


def alloc_workspace(T: int, N: int, K: int, device, path: int = PATH_AUTO) -> torch.Tensor:
    n = llmint8_workspace_bytes(T, N, K, path)
    if n == 0:
        raise ValueError(f"no workspace size for T={T} N={N} K={K} path={path}")
    return torch.empty(n, dtype=torch.uint8, device=device)


def llmint8_matmul(X: torch.Tensor, Wq: torch.Tensor, Wscale: torch.Tensor, W: torch.Tensor,
                   threshold: float = 6.0, workspace: torch.Tensor | None = None,
                   Y: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Y = X W^T by the LLM.int8() decomposition (fp16 [T,N])."""
    return llmint8_matmul_debug(X, Wq, Wscale, W, threshold, workspace, Y, PATH_AUTO, None,
                                stream, _entry="llmint8_matmul")


def llmint8_matmul_decode_noalloc(X: torch.Tensor, Wq: torch.Tensor, Wscale: torch.Tensor,
                                  W: torch.Tensor, threshold: float = 6.0,
                                  Y: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Decode-shaped Y = X W^T (T <= 16) with no workspace: the library's scratch
    is a fixed per-GPU array, for callers that must not allocate device memory.
    Calls must not overlap on the GPU (they share that array)."""
    _need(X, torch.float16, 2, "X")
    _need(Wq, torch.int8, 2, "Wq")
    _need(Wscale, torch.float32, 1, "Wscale")
    _need(W, torch.float16, 2, "W")
    T, K = X.shape
    N = Wq.shape[0]
    if Y is None:
        Y = torch.empty((T, N), dtype=torch.float16, device=X.device)
    _need(Y, torch.float16, 2, "Y")
    check_matmul_shapes(X, Wq, Wscale, W, Y)
    _check(load_library().llmint8_matmul_decode_noalloc(
        _ptr(X), T, K, _ptr(Wq), _ptr(Wscale), _ptr(W), N, float(threshold), _ptr(Y),
        _stream(stream)), "llmint8_matmul_decode_noalloc")
    return Y


def llmint8_int8_gemm_i32(Xq: torch.Tensor, Wq: torch.Tensor, acc: torch.Tensor | None = None,
                          stream=None) -> torch.Tensor:
    """acc = Xq Wq^T, exact int32 [T, N], on the library's tensor-core kernels
    (Xq int8 [T, K], Wq int8 [N, K])."""
    _need(Xq, torch.int8, 2, "Xq")
    _need(Wq, torch.int8, 2, "Wq")
    T, K = Xq.shape
    N = Wq.shape[0]
    if acc is None:
        acc = torch.empty((T, N), dtype=torch.int32, device=Xq.device)
    _need(acc, torch.int32, 2, "acc")
    if tuple(Wq.shape) != (N, K) or tuple(acc.shape) != (T, N) or Wq.device != Xq.device \
            or acc.device != Xq.device:
        raise ValueError(f"Wq must be [{N}, {K}] and acc [{T}, {N}] on {Xq.device}")
    _check(load_library().llmint8_int8_gemm_i32(_ptr(Xq), _ptr(Wq), T, N, K, _ptr(acc), _stream(stream)),
           "llmint8_int8_gemm_i32")
    return acc


def llmint8_matmul_debug(X, Wq, Wscale, W, threshold=6.0, workspace=None, Y=None,
                         path: int = PATH_AUTO, acc_out: torch.Tensor | None = None,
                         stream=None, _entry: str = "llmint8_matmul_debug",
                         xq_out: torch.Tensor | None = None, sx_out: torch.Tensor | None = None,
                         idx_out: torch.Tensor | None = None, n_out: torch.Tensor | None = None):
    _need(X, torch.float16, 2, "X")
    _need(Wq, torch.int8, 2, "Wq")
    _need(Wscale, torch.float32, 1, "Wscale")
    _need(W, torch.float16, 2, "W")
    T, K = X.shape
    N = Wq.shape[0]
    if Y is None:
        Y = torch.empty((T, N), dtype=torch.float16, device=X.device)
    _need(Y, torch.float16, 2, "Y")
    if acc_out is not None:
        _need(acc_out, torch.int32, 2, "acc_out")
    for t, dt, nd, name in ((xq_out, torch.int8, 2, "xq_out"), (sx_out, torch.float32, 1, "sx_out"),
                            (idx_out, torch.int32, 1, "idx_out"), (n_out, torch.int32, 1, "n_out")):
        if t is not None:
            _need(t, dt, nd, name)
    check_matmul_shapes(X, Wq, Wscale, W, Y, acc_out, xq_out, sx_out, idx_out, n_out)
    if workspace is None:
        workspace = alloc_workspace(T, N, K, X.device, path)
    else:
        _need(workspace, torch.uint8, 1, "workspace")
    lib = load_library()
    st = _stream(stream)
    if _entry == "llmint8_matmul":
        rc = lib.llmint8_matmul(_ptr(X), T, K, _ptr(Wq), _ptr(Wscale), _ptr(W), N,
                                float(threshold), _ptr(Y), _ptr(workspace), workspace.numel(), st)
    else:
        rc = lib.llmint8_matmul_debug(_ptr(X), T, K, _ptr(Wq), _ptr(Wscale), _ptr(W), N,
                                      float(threshold), _ptr(Y), _ptr(workspace),
                                      workspace.numel(), int(path), _ptr(acc_out), _ptr(xq_out),
                                      _ptr(sx_out), _ptr(idx_out), _ptr(n_out), st)
    _check(rc, _entry)
    return Y


def llmint8_matmul_profile(X, Wq, Wscale, W, threshold, workspace, Y, ev_begin, ev_end,
                           repeat: int = 1, path: int = PATH_AUTO, stream=None):
    """Activation stages once, then torch.cuda.Events around `repeat` launches
    of the main kernel."""
    for t, dt, nd, name in ((X, torch.float16, 2, "X"), (Wq, torch.int8, 2, "Wq"),
                            (Wscale, torch.float32, 1, "Wscale"), (W, torch.float16, 2, "W"),
                            (Y, torch.float16, 2, "Y"), (workspace, torch.uint8, 1, "workspace")):
        _need(t, dt, nd, name)
    check_matmul_shapes(X, Wq, Wscale, W, Y)
    T, K = X.shape
    N = Wq.shape[0]
    for ev in (ev_begin, ev_end):
        if ev.cuda_event == 0:  # torch creates the CUDA event on its first record
            ev.record()
    rc = load_library().llmint8_matmul_profile(
        _ptr(X), T, K, _ptr(Wq), _ptr(Wscale), _ptr(W), N, float(threshold), _ptr(Y),
        _ptr(workspace), workspace.numel(), int(path), int(repeat), ctypes.c_void_p(ev_begin.cuda_event),
        ctypes.c_void_p(ev_end.cuda_event), _stream(stream))
    _check(rc, "llmint8_matmul_profile")
    return Y


def llmint8_matmul_intermediates(X, Wq, Wscale, W, threshold=6.0, path: int = PATH_AUTO,
                                 workspace=None):
    """One llmint8_matmul_debug call returning (Y, acc, Xq, sx, outlier_idx)."""
    T, K = X.shape
    N = Wq.shape[0]
    dev = X.device
    acc = torch.empty((T, N), dtype=torch.int32, device=dev)
    Xq = torch.empty((T, K), dtype=torch.int8, device=dev)
    sx = torch.empty(T, dtype=torch.float32, device=dev)
    idx = torch.empty(K, dtype=torch.int32, device=dev)
    n = torch.zeros(1, dtype=torch.int32, device=dev)
    Y = llmint8_matmul_debug(X, Wq, Wscale, W, threshold, workspace, None, path, acc,
                             xq_out=Xq, sx_out=sx, idx_out=idx, n_out=n)
    return Y, acc, Xq, sx, idx[: int(n.item())]


def llmint8_detect_quantize(X: torch.Tensor, threshold: float = 6.0, path: int = PATH_AUTO,
                            workspace: torch.Tensor | None = None, stream=None):
    """Activation kernels of `path` alone -> (Xq int8 [T,K], xscale fp32 [T],
    outlier_idx int32 [|O|])."""
    _need(X, torch.float16, 2, "X")
    T, K = X.shape
    dev = X.device
    Xq = torch.empty((T, K), dtype=torch.int8, device=dev)
    sx = torch.empty(T, dtype=torch.float32, device=dev)
    idx = torch.empty(K, dtype=torch.int32, device=dev)
    n = torch.zeros(1, dtype=torch.int32, device=dev)
    if workspace is None:
        workspace = alloc_workspace(T, 0, K, dev, path)
    _check(load_library().llmint8_detect_quantize(
        _ptr(X), T, K, float(threshold), _ptr(Xq), _ptr(sx), _ptr(idx), _ptr(n),
        _ptr(workspace), workspace.numel(), int(path), _stream(stream)), "llmint8_detect_quantize")
    return Xq, sx, idx[: int(n.item())]


# ------------------------------------------------------------------ stored outlier columns

def llmint8_outlier_store_build(W: torch.Tensor, cols: torch.Tensor, stream=None):
    """(slot int32 [K], Wst fp16 [len(cols), N]): fp16 copies of the columns
    `cols` of W (int32, distinct, in [0, K)), one column per row of Wst."""
    _need(W, torch.float16, 2, "W")
    _need(cols, torch.int32, 1, "cols")
    N, K = W.shape
    if cols.device != W.device or cols.numel() > K:
        raise ValueError(f"cols must be at most {K} columns on {W.device}")
    slot = torch.empty(K, dtype=torch.int32, device=W.device)
    Wst = torch.empty((max(cols.numel(), 1), N), dtype=torch.float16, device=W.device)
    _check(load_library().llmint8_outlier_store_build(_ptr(W), N, K, _ptr(cols), cols.numel(), _ptr(slot),
                                                      _ptr(Wst), _stream(stream)), "llmint8_outlier_store_build")
    return slot, Wst


def llmint8_matmul_stored(X: torch.Tensor, Wq: torch.Tensor, Wscale: torch.Tensor, slot: torch.Tensor,
                          Wst: torch.Tensor, threshold: float = 6.0, workspace: torch.Tensor | None = None,
                          Y: torch.Tensor | None = None, n_miss: torch.Tensor | None = None, path: int = PATH_AUTO,
                          acc_out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Y = X W^T by the LLM.int8() decomposition with the outlier weights read
    from a column store (no fp16 W).  n_miss (int32 [1], optional) receives the
    number of outlier columns the store did not hold."""
    _need(X, torch.float16, 2, "X")
    _need(Wq, torch.int8, 2, "Wq")
    _need(Wscale, torch.float32, 1, "Wscale")
    _need(slot, torch.int32, 1, "slot")
    _need(Wst, torch.float16, 2, "Wst")
    T, K = X.shape
    N = Wq.shape[0]
    if Y is None:
        Y = torch.empty((T, N), dtype=torch.float16, device=X.device)
    _need(Y, torch.float16, 2, "Y")
    if acc_out is not None:
        _need(acc_out, torch.int32, 2, "acc_out")
    check_matmul_shapes(X, Wq, Wscale, None, Y, acc_out)
    if tuple(slot.shape) != (K,) or Wst.shape[1] != N or slot.device != X.device or Wst.device != X.device:
        raise ValueError(f"slot must be [{K}] and Wst [n, {N}] on {X.device}")
    if n_miss is not None:
        _need(n_miss, torch.int32, 1, "n_miss")
        if n_miss.numel() != 1 or n_miss.device != X.device:
            raise ValueError("n_miss must be one int32 on the device of X")
    if workspace is None:
        workspace = alloc_workspace(T, N, K, X.device, path)
    _need(workspace, torch.uint8, 1, "workspace")
    lib = load_library()
    if path != PATH_AUTO or acc_out is not None:
        rc = lib.llmint8_matmul_stored_debug(_ptr(X), T, K, _ptr(Wq), _ptr(Wscale), _ptr(slot), _ptr(Wst), N,
                                             float(threshold), _ptr(Y), _ptr(n_miss), _ptr(workspace),
                                             workspace.numel(), int(path), _ptr(acc_out), _stream(stream))
    else:
        rc = lib.llmint8_matmul_stored(_ptr(X), T, K, _ptr(Wq), _ptr(Wscale), _ptr(slot), _ptr(Wst), N,
                                       float(threshold), _ptr(Y), _ptr(n_miss), _ptr(workspace), workspace.numel(),
                                       _stream(stream))
    _check(rc, "llmint8_matmul_stored")
    return Y


# ------------------------------------------------------------------ FP8 E4M3

def llmint8_fp8_quantize_weight(W: torch.Tensor, stream=None):
    """W fp16 [N,K] -> (E4M3 codes uint8 [N,K], Wscale fp32 [N] = max|W[n]| / 448)."""
    _need(W, torch.float16, 2, "W")
    N, K = W.shape
    Wq = torch.empty((N, K), dtype=torch.uint8, device=W.device)
    Wscale = torch.empty(N, dtype=torch.float32, device=W.device)
    _check(load_library().llmint8_fp8_quantize_weight(_ptr(W), N, K, _ptr(Wq), _ptr(Wscale), _stream(stream)),
           "llmint8_fp8_quantize_weight")
    return Wq, Wscale


def llmint8_fp8_matmul(X: torch.Tensor, Wq: torch.Tensor, Wscale: torch.Tensor, W: torch.Tensor,
                       threshold: float = 6.0, workspace: torch.Tensor | None = None, Y: torch.Tensor | None = None,
                       path: int = PATH_AUTO, acc_out=None, xq_out=None, sx_out=None, idx_out=None, n_out=None,
                       stream=None) -> torch.Tensor:
    """Y = X W^T by the decomposition with E4M3 codes (fp16 [T,N])."""
    _need(X, torch.float16, 2, "X")
    _need(Wq, torch.uint8, 2, "Wq")
    _need(Wscale, torch.float32, 1, "Wscale")
    _need(W, torch.float16, 2, "W")
    T, K = X.shape
    N = Wq.shape[0]
    if Y is None:
        Y = torch.empty((T, N), dtype=torch.float16, device=X.device)
    _need(Y, torch.float16, 2, "Y")
    for t, dt, nd, name in ((acc_out, torch.float32, 2, "acc_out"), (xq_out, torch.uint8, 2, "xq_out"),
                            (sx_out, torch.float32, 1, "sx_out"), (idx_out, torch.int32, 1, "idx_out"),
                            (n_out, torch.int32, 1, "n_out")):
        if t is not None:
            _need(t, dt, nd, name)
    check_matmul_shapes(X, Wq, Wscale, W, Y, acc_out, xq_out, sx_out, idx_out, n_out)
    if workspace is None:
        workspace = alloc_workspace(T, N, K, X.device, path)
    _need(workspace, torch.uint8, 1, "workspace")
    lib = load_library()
    debug = path != PATH_AUTO or any(t is not None for t in (acc_out, xq_out, sx_out, idx_out, n_out))
    if debug:
        rc = lib.llmint8_fp8_matmul_debug(_ptr(X), T, K, _ptr(Wq), _ptr(Wscale), _ptr(W), N, float(threshold),
                                          _ptr(Y), _ptr(workspace), workspace.numel(), int(path), _ptr(acc_out),
                                          _ptr(xq_out), _ptr(sx_out), _ptr(idx_out), _ptr(n_out), _stream(stream))
    else:
        rc = lib.llmint8_fp8_matmul(_ptr(X), T, K, _ptr(Wq), _ptr(Wscale), _ptr(W), N, float(threshold), _ptr(Y),
                                    _ptr(workspace), workspace.numel(), _stream(stream))
    _check(rc, "llmint8_fp8_matmul")
    return Y


# ------------------------------------------------------------------ SmoothQuant W8A8

def llmint8_column_absmax(A: torch.Tensor, amax: torch.Tensor | None = None, accumulate: bool = False,
                          stream=None) -> torch.Tensor:
    """max over rows of |A[:, k]| (float32 [K]) of an fp16 matrix; with
    accumulate=True, folded into the existing amax."""
    _need(A, torch.float16, 2, "A")
    rows, K = A.shape
    if amax is None:
        if accumulate:
            raise ValueError("accumulate needs an existing amax")
        amax = torch.empty(K, dtype=torch.float32, device=A.device)
    _need(amax, torch.float32, 1, "amax")
    if tuple(amax.shape) != (K,) or amax.device != A.device:
        raise ValueError(f"amax must be [{K}] on {A.device}")
    _check(load_library().llmint8_column_absmax(_ptr(A), rows, K, _ptr(amax), int(bool(accumulate)),
                                                _stream(stream)), "llmint8_column_absmax")
    return amax


def llmint8_smooth_factors(ax: torch.Tensor, aw: torch.Tensor, alpha: float = 0.5, s: torch.Tensor | None = None,
                           stream=None) -> torch.Tensor:
    """s = ax^alpha / aw^(1 - alpha) per channel (1 where either maximum is 0)."""
    _need(ax, torch.float32, 1, "ax")
    _need(aw, torch.float32, 1, "aw")
    K = ax.shape[0]
    if s is None:
        s = torch.empty(K, dtype=torch.float32, device=ax.device)
    _need(s, torch.float32, 1, "s")
    if aw.shape != ax.shape or s.shape != ax.shape or aw.device != ax.device or s.device != ax.device:
        raise ValueError("ax, aw and s must have one shape and device")
    _check(load_library().llmint8_smooth_factors(_ptr(ax), _ptr(aw), K, float(alpha), _ptr(s), _stream(stream)),
           "llmint8_smooth_factors")
    return s


def llmint8_smoothquant_quantize_weight(W: torch.Tensor, s: torch.Tensor, stream=None):
    """W diag(s) quantised per output channel -> (Wq int8 [N,K], Wscale fp32 [N])."""
    _need(W, torch.float16, 2, "W")
    _need(s, torch.float32, 1, "s")
    N, K = W.shape
    if tuple(s.shape) != (K,) or s.device != W.device:
        raise ValueError(f"s must be [{K}] on {W.device}")
    Wq = torch.empty((N, K), dtype=torch.int8, device=W.device)
    Wscale = torch.empty(N, dtype=torch.float32, device=W.device)
    _check(load_library().llmint8_smoothquant_quantize_weight(_ptr(W), N, K, _ptr(s), _ptr(Wq), _ptr(Wscale),
                                                              _stream(stream)), "llmint8_smoothquant_quantize_weight")
    return Wq, Wscale


def llmint8_smoothquant_matmul(X: torch.Tensor, s: torch.Tensor, Wq: torch.Tensor, Wscale: torch.Tensor,
                               workspace: torch.Tensor | None = None, Y: torch.Tensor | None = None,
                               path: int = PATH_AUTO, acc_out=None, xq_out=None, sx_out=None,
                               stream=None) -> torch.Tensor:
    """Y = X W^T by SmoothQuant W8A8 (fp16 [T,N]) with the smoothed weight (Wq, Wscale)."""
    _need(X, torch.float16, 2, "X")
    _need(s, torch.float32, 1, "s")
    _need(Wq, torch.int8, 2, "Wq")
    _need(Wscale, torch.float32, 1, "Wscale")
    T, K = X.shape
    N = Wq.shape[0]
    if Y is None:
        Y = torch.empty((T, N), dtype=torch.float16, device=X.device)
    _need(Y, torch.float16, 2, "Y")
    for t, dt, nd, name in ((acc_out, torch.int32, 2, "acc_out"), (xq_out, torch.int8, 2, "xq_out"),
                            (sx_out, torch.float32, 1, "sx_out")):
        if t is not None:
            _need(t, dt, nd, name)
    check_matmul_shapes(X, Wq, Wscale, None, Y, acc_out, xq_out, sx_out)
    if tuple(s.shape) != (K,) or s.device != X.device:
        raise ValueError(f"s must be [{K}] on {X.device}")
    lib = load_library()
    if workspace is None:
        workspace = torch.empty(int(lib.llmint8_smoothquant_workspace_bytes(T, K)), dtype=torch.uint8,
                                device=X.device)
    _need(workspace, torch.uint8, 1, "workspace")
    debug = path != PATH_AUTO or acc_out is not None or xq_out is not None or sx_out is not None
    if debug:
        rc = lib.llmint8_smoothquant_matmul_debug(_ptr(X), T, K, _ptr(s), _ptr(Wq), _ptr(Wscale), N, _ptr(Y),
                                                  _ptr(workspace), workspace.numel(), int(path), _ptr(acc_out),
                                                  _ptr(xq_out), _ptr(sx_out), _stream(stream))
    else:
        rc = lib.llmint8_smoothquant_matmul(_ptr(X), T, K, _ptr(s), _ptr(Wq), _ptr(Wscale), N, _ptr(Y),
                                            _ptr(workspace), workspace.numel(), _stream(stream))
    _check(rc, "llmint8_smoothquant_matmul")
    return Y


def llmint8_sync_status(stream=None) -> int:
    """Wait for the stream; return the status in this device's error word (and clear it)."""
    return int(load_library().llmint8_sync_status(_stream(stream)))


def llmint8_selftest_timeout(wait_ns: int, stream=None):
    _check(load_library().llmint8_selftest_timeout(int(wait_ns), _stream(stream)),
           "llmint8_selftest_timeout")


class Int8Linear:
    """y = x W^T with W quantised once (per output channel) at construction.

    By default it holds Wq, Wscale and the fp16 W (read only at outlier
    columns).  With `store_columns` (a list of input columns, such as the
    outlier columns a calibration batch showed), it keeps fp16 copies of those
    columns only and drops the fp16 W: the resident weight is then about N*K
    bytes instead of 3*N*K; an outlier column outside the store uses the fp16
    value of its int8 weight and is counted in `last_misses`.  One workspace,
    sized for the largest T seen, is reused.
    """

    def __init__(self, W: torch.Tensor, threshold: float = 6.0, store_columns=None):
        W = W.contiguous()
        self.N, self.K = W.shape
        self.Wq, self.Wscale = llmint8_quantize_weight(W)
        self.threshold = float(threshold)
        self._ws = None
        if store_columns is None:
            self.W, self.slot, self.Wst, self._miss = W, None, None, None
        else:
            cols = torch.as_tensor(store_columns, dtype=torch.int32).to(W.device)
            self.slot, self.Wst = llmint8_outlier_store_build(W, cols)
            self.W = None
            self._miss = torch.zeros(1, dtype=torch.int32, device=W.device)

    def resident_weight_bytes(self) -> int:
        n = self.Wq.numel() + 4 * self.Wscale.numel()
        if self.W is not None:
            return n + 2 * self.W.numel()
        return n + 2 * self.Wst.numel() + 4 * self.slot.numel()

    @property
    def last_misses(self) -> int:
        """Outlier columns of the last call that the store did not hold (0 without a store)."""
        return 0 if self._miss is None else int(self._miss.item())

    def __call__(self, X: torch.Tensor) -> torch.Tensor:
        T, K = X.shape
        need = llmint8_workspace_bytes(T, self.N, K)
        if self._ws is None or self._ws.numel() < need:
            self._ws = torch.empty(need, dtype=torch.uint8, device=X.device)
        if self.W is None:
            return llmint8_matmul_stored(X, self.Wq, self.Wscale, self.slot, self.Wst, self.threshold, self._ws,
                                         n_miss=self._miss)
        return llmint8_matmul(X, self.Wq, self.Wscale, self.W, self.threshold, self._ws)
