"""CPU oracle for the LLM.int8() mixed-precision decomposition matmul.

TEST INFRASTRUCTURE.  Only the tests, the smoke check and the CPU-baseline leg
of the benchmark may import this module.  The CUDA product path never calls
it, and the two share no code: this wrapper loads `liboracle.so`, built from
`llmint8_oracle.c` with gcc, and passes numpy arrays by pointer.

Method (pages on LLM quantization, sections theirs):
  * 'LLM quantization, part 2' (hncyxsy.com) §2.1: per-output-feature weight
    scales (vector-wise quantization); feature dims whose activations reach the
    threshold 6.0 are outliers; their columns of X and W are multiplied in fp16;
    the rest in int8; the two partial products are summed.
  * '三、模型量化' (lowentro.cn) Q2: symmetric q = round(r/s),
    s = max|r| / (2^(b-1) - 1), r' = s*q.  Q4: the same decomposition.
  * '量化压缩实战' (tqpw.cn) §2.1: scale = max_val/127, round, clip; worked
    example [0.0023,-1.5,4.7,0.001,8.9,-2.3] -> [0,-21,67,0,127,-33].

Readings where the pages are silent or ambiguous:
outlier test |x| >= tau on any row of this call; per-row activation scale over
the non-outlier columns; weight scale over all columns; round half to even in
binary32 on fl(x/s); clamp to [-127, 127]; s = 0 gives code 0; the fp part and
the sum in binary64, rounded once to fp16.

Pinned by tests/test_oracle.py against the pages' worked example, closed forms,
textbook special cases (tau = 0 is an fp16 GEMM, tau = inf is a plain int8
GEMM, integer inputs quantise exactly), brute-force fp64 with the quantisation
error bound, and invariants.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "llmint8_oracle.c")
_LIBPATH = os.path.join(_HERE, "liboracle.so")
_LOCK = threading.Lock()
_LIB = None

CFLAGS = ["-O2", "-std=c11", "-fno-fast-math", "-ffp-contract=off", "-fopenmp", "-fPIC",
           "-shared", "-Wall", "-Wextra"]


def build(force: bool = False) -> str:
    """Compile liboracle.so next to its source (gcc, OpenMP).  With
    LLMINT8_ORACLE_LIB set, that library is used as it is instead: the
    mutation tests compile copies of the source with planted mistakes and run
    the pins against them."""
    override = os.environ.get("LLMINT8_ORACLE_LIB")
    if override:
        return override
    if force or not os.path.exists(_LIBPATH) or os.path.getmtime(_LIBPATH) < max(
            os.path.getmtime(_SRC), os.path.getmtime(os.path.join(_HERE, "llmint8_oracle.h"))):
        tmp = _LIBPATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *CFLAGS, "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIBPATH)
    return _LIBPATH


def _lib():
    global _LIB
    with _LOCK:
        if _LIB is None:
            lib = ctypes.CDLL(build())
            P, I64, F, I = ctypes.c_void_p, ctypes.c_int64, ctypes.c_float, ctypes.c_int
            sig = {
                "oracle_h2f_array": (None, [P, I64, P]),
                "oracle_d2h_array": (None, [P, I64, P]),
                "oracle_quantize_weight": (None, [P, I64, I64, P, P]),
                "oracle_detect_outliers": (None, [P, I64, I64, F, P]),
                "oracle_compact": (I64, [P, I64, P]),
                "oracle_quantize_activations": (None, [P, I64, I64, P, P, P]),
                "oracle_int8_gemm": (I, [P, P, I64, I64, I64, P]),
                "oracle_outlier_gemm": (None, [P, P, I64, I64, I64, P, I64, P]),
                "oracle_dequant_combine": (None, [P, P, P, P, I64, I64, P]),
                "oracle_matmul": (I, [P, I64, I64, P, P, P, I64, F, P, P, P, P, P, P, P, P]),
                "oracle_num_threads": (I, []),
            }
            for name, (res, args) in sig.items():
                fn = getattr(lib, name)
                fn.restype = res
                fn.argtypes = args
            _LIB = lib
    return _LIB


def _p(a: np.ndarray | None):
    return None if a is None else ctypes.c_void_p(a.ctypes.data)


def _bits(a: np.ndarray) -> np.ndarray:
    a = np.ascontiguousarray(a)
    if a.dtype == np.float16:
        return a.view(np.uint16)
    assert a.dtype == np.uint16, a.dtype
    return a


def num_threads() -> int:
    return int(_lib().oracle_num_threads())


def h2f(h: np.ndarray) -> np.ndarray:
    h = _bits(h)
    out = np.empty(h.shape, np.float32)
    _lib().oracle_h2f_array(_p(h), h.size, _p(out))
    return out


def d2h(v: np.ndarray) -> np.ndarray:
    """binary64 values -> fp16 (returned as np.float16), nearest-even."""
    v = np.ascontiguousarray(v, dtype=np.float64)
    out = np.empty(v.shape, np.uint16)
    _lib().oracle_d2h_array(_p(v), v.size, _p(out))
    return out.view(np.float16)


def quantize_weight(W: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """a0: Wq int8 [N,K], sw float32 [N]."""
    Wb = _bits(W)
    N, K = Wb.shape
    Wq = np.empty((N, K), np.int8)
    sw = np.empty(N, np.float32)
    _lib().oracle_quantize_weight(_p(Wb), N, K, _p(Wq), _p(sw))
    return Wq, sw


def detect_outliers(X: np.ndarray, tau: float) -> np.ndarray:
    """a1: flag uint8 [K]."""
    Xb = _bits(X)
    T, K = Xb.shape
    flag = np.empty(K, np.uint8)
    _lib().oracle_detect_outliers(_p(Xb), T, K, float(tau), _p(flag))
    return flag


def compact(flag: np.ndarray) -> np.ndarray:
    """a4: ascending int32 outlier indices."""
    flag = np.ascontiguousarray(flag, dtype=np.uint8)
    idx = np.empty(max(flag.size, 1), np.int32)
    n = _lib().oracle_compact(_p(flag), flag.size, _p(idx))
    return idx[:n].copy()


def quantize_activations(X: np.ndarray, flag: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """a2+a3: Xq int8 [T,K], sx float32 [T]."""
    Xb = _bits(X)
    T, K = Xb.shape
    flag = np.ascontiguousarray(flag, dtype=np.uint8)
    Xq = np.empty((T, K), np.int8)
    sx = np.empty(T, np.float32)
    _lib().oracle_quantize_activations(_p(Xb), T, K, _p(flag), _p(Xq), _p(sx))
    return Xq, sx


def int8_gemm(Xq: np.ndarray, Wq: np.ndarray) -> np.ndarray:
    """a5: int32 [T,N]; raises if a sum leaves int32."""
    Xq = np.ascontiguousarray(Xq, dtype=np.int8)
    Wq = np.ascontiguousarray(Wq, dtype=np.int8)
    T, K = Xq.shape
    N, K2 = Wq.shape
    assert K == K2
    acc = np.empty((T, N), np.int32)
    rc = _lib().oracle_int8_gemm(_p(Xq), _p(Wq), T, N, K, _p(acc))
    if rc != 0:
        raise OverflowError("int8 GEMM sum does not fit int32")
    return acc


def outlier_gemm(X: np.ndarray, W: np.ndarray, idx: np.ndarray) -> np.ndarray:
    """a6: binary64 [T,N] product over the outlier columns."""
    Xb, Wb = _bits(X), _bits(W)
    T, K = Xb.shape
    N = Wb.shape[0]
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    yo = np.empty((T, N), np.float64)
    _lib().oracle_outlier_gemm(_p(Xb), _p(Wb), T, N, K, _p(idx) if idx.size else None,
                               idx.size, _p(yo))
    return yo


def dequant_combine(acc, sx, sw, yo) -> np.ndarray:
    """a7: Y fp16 [T,N]."""
    acc = np.ascontiguousarray(acc, dtype=np.int32)
    sx = np.ascontiguousarray(sx, dtype=np.float32)
    sw = np.ascontiguousarray(sw, dtype=np.float32)
    T, N = acc.shape
    if yo is not None:
        yo = np.ascontiguousarray(yo, dtype=np.float64)
    Y = np.empty((T, N), np.uint16)
    _lib().oracle_dequant_combine(_p(acc), _p(sx), _p(sw), _p(yo), T, N, _p(Y))
    return Y.view(np.float16)


def matmul(X: np.ndarray, Wq: np.ndarray, sw: np.ndarray, W: np.ndarray, tau: float,
           intermediates: bool = False):
    """a1..a7: Y fp16 [T,N]; with intermediates=True also a dict of every stage."""
    Xb, Wb = _bits(X), _bits(W)
    T, K = Xb.shape
    N = Wb.shape[0]
    Wq = np.ascontiguousarray(Wq, dtype=np.int8)
    sw = np.ascontiguousarray(sw, dtype=np.float32)
    Y = np.empty((T, N), np.uint16)
    flag = np.empty(K, np.uint8)
    idx = np.empty(max(K, 1), np.int32)
    nO = ctypes.c_int64(0)
    Xq = np.empty((T, K), np.int8)
    sx = np.empty(T, np.float32)
    acc = np.empty((T, N), np.int32)
    yo = np.empty((T, N), np.float64)
    rc = _lib().oracle_matmul(_p(Xb), T, K, _p(Wq), _p(sw), _p(Wb), N, float(tau), _p(Y),
                              _p(flag), _p(idx), ctypes.byref(nO), _p(Xq), _p(sx), _p(acc),
                              _p(yo))
    if rc == -1:
        raise OverflowError("int8 GEMM sum does not fit int32")
    if rc != 0:
        raise MemoryError("oracle allocation failed")
    Y = Y.view(np.float16)
    if not intermediates:
        return Y
    return Y, dict(flag=flag, idx=idx[: nO.value].copy(), nO=int(nO.value), Xq=Xq, sx=sx,
                   acc=acc, yo=yo)
