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
    _check(load_library().llmint8_matmul_decode_noalloc(
        _ptr(X), T, K, _ptr(Wq), _ptr(Wscale), _ptr(W), N, float(threshold), _ptr(Y),
        _stream(stream)), "llmint8_matmul_decode_noalloc")
    return Y


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
    if Wq.shape != (N, K) or W.shape != (N, K) or Wscale.shape != (N,):
        raise ValueError("shape mismatch between X, Wq, Wscale and W")
    if Y is None:
        Y = torch.empty((T, N), dtype=torch.float16, device=X.device)
    _need(Y, torch.float16, 2, "Y")
    if workspace is None:
        workspace = alloc_workspace(T, N, K, X.device, path)
    if acc_out is not None:
        _need(acc_out, torch.int32, 2, "acc_out")
    for t, dt, nd, name in ((xq_out, torch.int8, 2, "xq_out"), (sx_out, torch.float32, 1, "sx_out"),
                            (idx_out, torch.int32, 1, "idx_out"), (n_out, torch.int32, 1, "n_out")):
        if t is not None:
            _need(t, dt, nd, name)
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


def llmint8_sync_status(stream=None) -> int:
    """Wait for the stream; return the status in this device's error word (and clear it)."""
    return int(load_library().llmint8_sync_status(_stream(stream)))


def llmint8_selftest_timeout(wait_ns: int, stream=None):
    _check(load_library().llmint8_selftest_timeout(int(wait_ns), _stream(stream)),
           "llmint8_selftest_timeout")


class Int8Linear:
    """y = x W^T with W quantised once (per output channel) at construction.

    Holds Wq, Wscale and the fp16 W (read only at outlier columns), and reuses
    one workspace sized for the largest T seen.
    """

    def __init__(self, W: torch.Tensor, threshold: float = 6.0):
        self.W = W.contiguous()
        self.Wq, self.Wscale = llmint8_quantize_weight(self.W)
        self.threshold = float(threshold)
        self._ws = None

    def __call__(self, X: torch.Tensor) -> torch.Tensor:
        T, K = X.shape
        need = llmint8_workspace_bytes(T, self.W.shape[0], K)
        if self._ws is None or self._ws.numel() < need:
            self._ws = torch.empty(need, dtype=torch.uint8, device=X.device)
        return llmint8_matmul(X, self.Wq, self.Wscale, self.W, self.threshold, self._ws)
