"""CPU oracle for the variants built on the LLM.int8() path: SmoothQuant W8A8,
the FP8 (E4M3) decomposition and the decomposition with stored outlier-weight
columns.

TEST INFRASTRUCTURE.  Only the tests, the smoke check and the CPU-baseline leg
of the benchmark may import this module; the CUDA product path never calls it
and shares no code with it.  It loads `liboracle_next.so`, compiled by gcc from
`next_oracle.c` together with the pinned `llmint8_oracle.c` (whose fp16
conversions, int8 codes, outlier detection and int8 product it reuses).

Sources and readings (pages on LLM quantization, sections theirs):
  * SmoothQuant -- 'LLM quantization, part 2' (hncyxsy.com) §5 and '三、模型量化'
    (lowentro.cn) Q9-Q10: Y = (X diag(s)^-1)(diag(s) W) exactly; s_j from the
    channel maxima with strength alpha.  The Q10 formula prints a product;
    the quotient max|X_j|^a / max|W_j|^(1-a) is the reading taken, because it
    is the one that balances both sides' ranges at a = 0.5 as Q10 says the
    factor should.  A channel with zero maximum on either side keeps s = 1.
  * FP8 -- '量化压缩实战' (tqpw.cn) §3.6: E4M3 codes (1/4/3 bits, largest finite
    448); absmax scales map the largest regular magnitude to 448; round to
    nearest even, saturating.
  * Stored outlier columns -- 'LLM quantization, part 2' §2.2 (8-bit weights
    for memory) with §2.1's fp16 outlier weights: fp16 weights are kept only
    for a set of columns; an outlier outside it uses fp16(fl(sw * q)) and is
    counted as a miss.

Pinned by tests/test_oracle_next.py.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

from oracle import oracle as base

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRCS = [os.path.join(_HERE, "llmint8_oracle.c"), os.path.join(_HERE, "next_oracle.c")]
_HDRS = [os.path.join(_HERE, "llmint8_oracle.h"), os.path.join(_HERE, "next_oracle.h")]
_LIBPATH = os.path.join(_HERE, "liboracle_next.so")
_LOCK = threading.Lock()
_LIB = None


def build(force: bool = False) -> str:
    """Compile liboracle_next.so (gcc, OpenMP).  LLMINT8_ORACLE_NEXT_LIB
    overrides it, for the mutation tests."""
    override = os.environ.get("LLMINT8_ORACLE_NEXT_LIB")
    if override:
        return override
    newest = max(os.path.getmtime(p) for p in _SRCS + _HDRS)
    if force or not os.path.exists(_LIBPATH) or os.path.getmtime(_LIBPATH) < newest:
        tmp = _LIBPATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *base.CFLAGS, "-o", tmp, *_SRCS, "-lm"])
        os.replace(tmp, _LIBPATH)
    return _LIBPATH


def _lib():
    global _LIB
    with _LOCK:
        if _LIB is None:
            lib = ctypes.CDLL(build())
            P, I64, F, I = ctypes.c_void_p, ctypes.c_int64, ctypes.c_float, ctypes.c_int
            sig = {
                "onext_column_absmax": (None, [P, I64, I64, P]),
                "onext_pow": (F, [F, F]),
                "onext_smooth_factors": (None, [P, P, I64, F, P]),
                "onext_smooth_quantize_weight": (None, [P, P, I64, I64, P, P]),
                "onext_smooth_quantize_activations": (None, [P, P, I64, I64, P, P]),
                "onext_smoothquant_matmul": (I, [P, P, I64, I64, P, P, I64, P, P, P, P]),
                "onext_e4m3_to_float": (F, [ctypes.c_uint8]),
                "onext_float_to_e4m3": (ctypes.c_uint8, [F]),
                "onext_quantize_e4m3": (ctypes.c_uint8, [F, F]),
                "onext_fp8_quantize_weight": (None, [P, I64, I64, P, P]),
                "onext_fp8_quantize_activations": (None, [P, I64, I64, P, P, P]),
                "onext_fp8_gemm": (None, [P, P, I64, I64, I64, P]),
                "onext_fp8_matmul": (I, [P, I64, I64, P, P, P, I64, F, P, P, P, P, P, P, P, P]),
                "onext_reconstruct_weight": (ctypes.c_uint16, [ctypes.c_int8, F]),
                "onext_outlier_gemm_stored": (I64, [P, P, P, P, P, I64, I64, I64, P, I64, P]),
                "onext_matmul_stored": (I, [P, I64, I64, P, P, P, P, I64, F, P, P]),
            }
            for name, (res, args) in sig.items():
                fn = getattr(lib, name)
                fn.restype = res
                fn.argtypes = args
            _LIB = lib
    return _LIB


def _p(a):
    return None if a is None else ctypes.c_void_p(a.ctypes.data)


_bits = base._bits


def _f32(a):
    return np.ascontiguousarray(a, dtype=np.float32)


# ------------------------------------------------------------------ SmoothQuant

def column_absmax(A: np.ndarray) -> np.ndarray:
    """max over rows of |A[:, k]| (float32 [K]) of an fp16 matrix."""
    Ab = _bits(A)
    rows, K = Ab.shape
    out = np.empty(K, np.float32)
    _lib().onext_column_absmax(_p(Ab), rows, K, _p(out))
    return out


def pow32(p: float, a: float) -> float:
    return float(_lib().onext_pow(float(p), float(a)))


def smooth_factors(ax: np.ndarray, aw: np.ndarray, alpha: float = 0.5) -> np.ndarray:
    ax, aw = _f32(ax), _f32(aw)
    s = np.empty(ax.size, np.float32)
    _lib().onext_smooth_factors(_p(ax), _p(aw), ax.size, float(alpha), _p(s))
    return s


def smooth_quantize_weight(W: np.ndarray, s: np.ndarray):
    Wb, s = _bits(W), _f32(s)
    N, K = Wb.shape
    Wq = np.empty((N, K), np.int8)
    sw = np.empty(N, np.float32)
    _lib().onext_smooth_quantize_weight(_p(Wb), _p(s), N, K, _p(Wq), _p(sw))
    return Wq, sw


def smooth_quantize_activations(X: np.ndarray, s: np.ndarray):
    Xb, s = _bits(X), _f32(s)
    T, K = Xb.shape
    Xq = np.empty((T, K), np.int8)
    sx = np.empty(T, np.float32)
    _lib().onext_smooth_quantize_activations(_p(Xb), _p(s), T, K, _p(Xq), _p(sx))
    return Xq, sx


def smoothquant_matmul(X, s, Wq, sw, intermediates: bool = False):
    Xb, s = _bits(X), _f32(s)
    T, K = Xb.shape
    Wq = np.ascontiguousarray(Wq, dtype=np.int8)
    sw = _f32(sw)
    N = Wq.shape[0]
    Y = np.empty((T, N), np.uint16)
    Xq = np.empty((T, K), np.int8)
    sx = np.empty(T, np.float32)
    acc = np.empty((T, N), np.int32)
    rc = _lib().onext_smoothquant_matmul(_p(Xb), _p(s), T, K, _p(Wq), _p(sw), N, _p(Y), _p(Xq), _p(sx), _p(acc))
    if rc == -1:
        raise OverflowError("int8 GEMM sum does not fit int32")
    if rc != 0:
        raise MemoryError("oracle allocation failed")
    Y = Y.view(np.float16)
    return (Y, dict(Xq=Xq, sx=sx, acc=acc)) if intermediates else Y


# ------------------------------------------------------------------ FP8 E4M3

_E4M3_TABLE = None


def e4m3_to_float(codes: np.ndarray) -> np.ndarray:
    """Values of E4M3 codes (float32), looked up in the table of all 256 codes
    that onext_e4m3_to_float decodes."""
    global _E4M3_TABLE
    if _E4M3_TABLE is None:
        f = _lib().onext_e4m3_to_float
        _E4M3_TABLE = np.array([f(v) for v in range(256)], np.float32)
    return _E4M3_TABLE[np.asarray(codes, dtype=np.uint8)]


def float_to_e4m3(x: np.ndarray) -> np.ndarray:
    f = _lib().onext_float_to_e4m3
    a = np.asarray(x, dtype=np.float32)
    return np.array([f(float(v)) for v in a.ravel()], np.uint8).reshape(a.shape)


def fp8_quantize_weight(W: np.ndarray):
    Wb = _bits(W)
    N, K = Wb.shape
    Wq = np.empty((N, K), np.uint8)
    sw = np.empty(N, np.float32)
    _lib().onext_fp8_quantize_weight(_p(Wb), N, K, _p(Wq), _p(sw))
    return Wq, sw


def fp8_quantize_activations(X: np.ndarray, flag: np.ndarray):
    Xb = _bits(X)
    T, K = Xb.shape
    flag = np.ascontiguousarray(flag, dtype=np.uint8)
    Xq = np.empty((T, K), np.uint8)
    sx = np.empty(T, np.float32)
    _lib().onext_fp8_quantize_activations(_p(Xb), T, K, _p(flag), _p(Xq), _p(sx))
    return Xq, sx


def fp8_gemm(Xq: np.ndarray, Wq: np.ndarray) -> np.ndarray:
    Xq = np.ascontiguousarray(Xq, dtype=np.uint8)
    Wq = np.ascontiguousarray(Wq, dtype=np.uint8)
    T, K = Xq.shape
    N = Wq.shape[0]
    acc = np.empty((T, N), np.float64)
    _lib().onext_fp8_gemm(_p(Xq), _p(Wq), T, N, K, _p(acc))
    return acc


def fp8_matmul(X, Wq, sw, W, tau: float, intermediates: bool = False):
    Xb, Wb = _bits(X), _bits(W)
    T, K = Xb.shape
    N = Wb.shape[0]
    Wq = np.ascontiguousarray(Wq, dtype=np.uint8)
    sw = _f32(sw)
    Y = np.empty((T, N), np.uint16)
    flag = np.empty(K, np.uint8)
    idx = np.empty(max(K, 1), np.int32)
    nO = ctypes.c_int64(0)
    Xq = np.empty((T, K), np.uint8)
    sx = np.empty(T, np.float32)
    acc = np.empty((T, N), np.float64)
    yo = np.empty((T, N), np.float64)
    rc = _lib().onext_fp8_matmul(_p(Xb), T, K, _p(Wq), _p(sw), _p(Wb), N, float(tau), _p(Y), _p(flag),
                                 _p(idx), ctypes.byref(nO), _p(Xq), _p(sx), _p(acc), _p(yo))
    if rc != 0:
        raise MemoryError("oracle allocation failed")
    Y = Y.view(np.float16)
    if not intermediates:
        return Y
    return Y, dict(flag=flag, idx=idx[: nO.value].copy(), nO=int(nO.value), Xq=Xq, sx=sx, acc=acc, yo=yo)


# ------------------------------------------------------------------ stored outlier columns

def reconstruct_weight(q: int, s: float) -> np.float16:
    return np.uint16(_lib().onext_reconstruct_weight(int(q), float(s))).view(np.float16)


def make_store(W: np.ndarray, cols) -> tuple[np.ndarray, np.ndarray]:
    """(slot int32 [K], Wst fp16 [len(cols)][N]): column cols[i] of W stored as
    row i of Wst; slot[k] = i for stored columns, -1 elsewhere."""
    N, K = W.shape
    cols = np.asarray(cols, dtype=np.int64)
    slot = np.full(K, -1, np.int32)
    slot[cols] = np.arange(cols.size, dtype=np.int32)
    Wst = np.ascontiguousarray(W[:, cols].T) if cols.size else np.zeros((0, N), np.float16)
    return slot, Wst


def outlier_gemm_stored(X, Wq, sw, slot, Wst, idx):
    Xb = _bits(X)
    T, K = Xb.shape
    Wq = np.ascontiguousarray(Wq, dtype=np.int8)
    N = Wq.shape[0]
    sw, slot = _f32(sw), np.ascontiguousarray(slot, dtype=np.int32)
    Wst = _bits(Wst) if Wst.size else np.zeros((1, N), np.uint16)
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    yo = np.empty((T, N), np.float64)
    miss = _lib().onext_outlier_gemm_stored(_p(Xb), _p(Wq), _p(sw), _p(slot), _p(Wst), T, N, K,
                                            _p(idx) if idx.size else None, idx.size, _p(yo))
    return yo, int(miss)


def matmul_stored(X, Wq, sw, slot, Wst, tau: float):
    """Y fp16 [T, N] and the miss count."""
    Xb = _bits(X)
    T, K = Xb.shape
    Wq = np.ascontiguousarray(Wq, dtype=np.int8)
    N = Wq.shape[0]
    sw, slot = _f32(sw), np.ascontiguousarray(slot, dtype=np.int32)
    Wst = _bits(Wst) if Wst.size else np.zeros((1, N), np.uint16)
    Y = np.empty((T, N), np.uint16)
    miss = ctypes.c_int64(0)
    rc = _lib().onext_matmul_stored(_p(Xb), T, K, _p(Wq), _p(sw), _p(slot), _p(Wst), N, float(tau), _p(Y),
                                    ctypes.byref(miss))
    if rc == -1:
        raise OverflowError("int8 GEMM sum does not fit int32")
    if rc != 0:
        raise MemoryError("oracle allocation failed")
    return Y.view(np.float16), int(miss.value)
