"""CPU oracle for the LLM.int8() decomposed matmul (ctypes wrapper over oracle.c).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import this package.  It
shares no code with the CUDA path and the CUDA path never calls it.

Each function restates one step of the method as the pages define it; the
citations are in ``oracle.c``.  Arrays are numpy: fp16 inputs as ``np.float16``
(passed to C as their raw binary16 bits), codes as ``int8``, scales as
``float32``, accumulators as ``int32``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")

CFLAGS = ["-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math", "-std=c11",
          "-shared", "-fPIC", "-Wall"]


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so next to it (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB_PATH) or \
            os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *CFLAGS, _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


_lib = None


def lib():
    global _lib
    if _lib is None:
        # INT8MM_ORACLE_LIB is set only by the oracle's own mutation test, to
        # run the pins against a copy of oracle.c with one planted mistake
        path = os.environ.get("INT8MM_ORACLE_LIB")
        if not path:
            path = build()
        L = ctypes.CDLL(path)
        P = ctypes.c_void_p
        I64 = ctypes.c_int64
        L.orc_half_to_double.argtypes = [ctypes.c_uint16]
        L.orc_half_to_double.restype = ctypes.c_double
        L.orc_double_to_half.argtypes = [ctypes.c_double]
        L.orc_double_to_half.restype = ctypes.c_uint16
        L.orc_half_to_double_array.argtypes = [P, I64, P]
        L.orc_double_to_half_array.argtypes = [P, I64, P]
        L.orc_scale_from_absmax.argtypes = [ctypes.c_float]
        L.orc_scale_from_absmax.restype = ctypes.c_float
        L.orc_quantize_value.argtypes = [ctypes.c_float, ctypes.c_float]
        L.orc_quantize_value.restype = ctypes.c_int8
        L.orc_outlier_columns.argtypes = [P, I64, I64, ctypes.c_float, P, P]
        L.orc_outlier_columns.restype = I64
        L.orc_quantize_rows.argtypes = [P, I64, I64, P, I64, P, P]
        L.orc_rebuild_weight_rows.argtypes = [P, P, I64, I64, P]
        L.orc_quantize_cols.argtypes = [P, I64, I64, P, P]
        L.orc_int8_matmul.argtypes = [P, P, I64, I64, I64, P]
        L.orc_int8_matmul.restype = ctypes.c_int
        L.orc_dequant_add_outliers.argtypes = [P, P, P, P, P, I64, I64, I64, P, I64, P, P, P]
        L.orc_matmul_f64.argtypes = [P, P, I64, I64, I64, P]
        L.orc_tensorwise_absmax.argtypes = [P, P, I64, I64, I64, P, P, P, P, P]
        L.orc_tensorwise_absmax.restype = ctypes.c_int
        L.orc_num_threads.restype = ctypes.c_int
        L.orc_set_num_threads.argtypes = [ctypes.c_int]
        _lib = L
    return _lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return ctypes.c_void_p(a.ctypes.data)


def _f16(a) -> np.ndarray:
    a = np.ascontiguousarray(a)
    assert a.dtype == np.float16, a.dtype
    return a


# --------------------------------------------------------------------------
# binary16 codec

def half_to_double(h: np.ndarray) -> np.ndarray:
    h = np.ascontiguousarray(h, dtype=np.uint16)
    out = np.empty(h.shape, np.float64)
    lib().orc_half_to_double_array(_p(h), h.size, _p(out))
    return out


def double_to_half(v: np.ndarray) -> np.ndarray:
    """Round doubles to binary16 (ties to even); returns the uint16 codes."""
    v = np.ascontiguousarray(v, dtype=np.float64)
    out = np.empty(v.shape, np.uint16)
    lib().orc_double_to_half_array(_p(v), v.size, _p(out))
    return out


def scale_from_absmax(a: float) -> np.float32:
    return np.float32(lib().orc_scale_from_absmax(float(np.float32(a))))


def quantize_value(x: float, c: float) -> int:
    return int(lib().orc_quantize_value(float(np.float32(x)), float(np.float32(c))))


# --------------------------------------------------------------------------
# the method, step by step

def outlier_columns(X: np.ndarray, alpha: float):
    """Step 1: colmax[K] (fp32) and the ascending outlier index list."""
    X = _f16(X)
    M, K = X.shape
    colmax = np.empty(K, np.float32)
    idx = np.empty(K, np.int32)
    n = lib().orc_outlier_columns(_p(X), M, K, float(np.float32(alpha)), _p(colmax), _p(idx))
    return colmax, idx[:n].copy()


def quantize_rows(X: np.ndarray, idx: np.ndarray):
    """Step 2a: int8 codes [M,K] (outlier columns 0) and c_x[M]."""
    X = _f16(X)
    M, K = X.shape
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    q = np.empty((M, K), np.int8)
    c = np.empty(M, np.float32)
    lib().orc_quantize_rows(_p(X), M, K, _p(idx), idx.size, _p(q), _p(c))
    return q, c


def quantize_cols(W: np.ndarray):
    """Step 2b: int8 codes [K,N] and c_w[N]."""
    W = _f16(W)
    K, N = W.shape
    q = np.empty((K, N), np.int8)
    c = np.empty(N, np.float32)
    lib().orc_quantize_cols(_p(W), K, N, _p(q), _p(c))
    return q, c


def rebuild_weight_rows(qw: np.ndarray, c_w: np.ndarray) -> np.ndarray:
    """W rebuilt from its codes, fp16(q * (1/c_w)) per element, [K, N]."""
    qw = np.ascontiguousarray(qw, dtype=np.int8)
    c_w = np.ascontiguousarray(c_w, dtype=np.float32)
    K, N = qw.shape
    out = np.empty((K, N), dtype=np.uint16)
    lib().orc_rebuild_weight_rows(_p(qw), _p(c_w), K, N, _p(out))
    return out.view(np.float16)


def static_weight(W: np.ndarray, qw: np.ndarray, c_w: np.ndarray, rows) -> np.ndarray:
    """The weight rows a memory-saving prepared weight uses in the outlier
    product: W[k] for the stored dimensions k in `rows`, the rebuilt row for
    every other k."""
    Ws = rebuild_weight_rows(qw, c_w)
    r = np.asarray(list(rows), dtype=np.int64)
    if r.size:
        Ws[r] = _f16(W)[r]
    return Ws


def int8_matmul(qx: np.ndarray, qw: np.ndarray) -> np.ndarray:
    """Step 3: int32 accumulator [M,N]; raises if a sum leaves int32."""
    qx = np.ascontiguousarray(qx, dtype=np.int8)
    qw = np.ascontiguousarray(qw, dtype=np.int8)
    M, K = qx.shape
    K2, N = qw.shape
    assert K == K2
    acc = np.empty((M, N), np.int32)
    if lib().orc_int8_matmul(_p(qx), _p(qw), M, K, N, _p(acc)) != 0:
        raise OverflowError("int8 contraction does not fit int32")
    return acc


def dequant_add_outliers(acc, c_x, c_w, X, W, idx, bias=None):
    """Steps 4-5 (plus the layer's optional fp16 bias [N]): fp16 Y [M,N] and
    the unrounded double value."""
    X = _f16(X)
    W = _f16(W)
    acc = np.ascontiguousarray(acc, dtype=np.int32)
    c_x = np.ascontiguousarray(c_x, dtype=np.float32)
    c_w = np.ascontiguousarray(c_w, dtype=np.float32)
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    M, K = X.shape
    N = W.shape[1]
    b = None if bias is None else _f16(np.asarray(bias).reshape(N))
    Y = np.empty((M, N), np.uint16)
    Yx = np.empty((M, N), np.float64)
    lib().orc_dequant_add_outliers(_p(acc), _p(c_x), _p(c_w), _p(X), _p(W), M, K, N,
                                   _p(idx), idx.size, None if b is None else _p(b), _p(Y), _p(Yx))
    return Y.view(np.float16), Yx


def decomp_matmul(X: np.ndarray, W: np.ndarray, alpha: float, rows=None, wq=None, bias=None):
    """The whole method.  Outlier detection always uses all rows of X; with
    ``rows`` given, only those rows of the output (and of the X codes) are
    computed.  ``wq`` may pass a previous ``quantize_cols(W)`` result;
    ``bias`` is the layer's optional fp16 bias [N]."""
    X = _f16(X)
    W = _f16(W)
    colmax, idx = outlier_columns(X, alpha)
    Xr = X if rows is None else np.ascontiguousarray(X[np.asarray(rows)])
    qx, c_x = quantize_rows(Xr, idx)
    qw, c_w = quantize_cols(W) if wq is None else wq
    acc = int8_matmul(qx, qw)
    Y, Yx = dequant_add_outliers(acc, c_x, c_w, Xr, W, idx, bias)
    return dict(colmax=colmax, idx=idx, qx=qx, c_x=c_x, qw=qw, c_w=c_w,
                acc=acc, Y=Y, Y_exact=Yx)


def matmul_f64(X: np.ndarray, W: np.ndarray) -> np.ndarray:
    X = _f16(X)
    W = _f16(W)
    M, K = X.shape
    N = W.shape[1]
    Y = np.empty((M, N), np.float64)
    lib().orc_matmul_f64(_p(X), _p(W), M, K, N, _p(Y))
    return Y


def tensorwise_absmax(X: np.ndarray, W: np.ndarray):
    """Comparator: one absmax scale per tensor, no decomposition."""
    X = _f16(X)
    W = _f16(W)
    M, K = X.shape
    N = W.shape[1]
    qx = np.empty((M, K), np.int8)
    qw = np.empty((K, N), np.int8)
    cx = np.empty(1, np.float32)
    cw = np.empty(1, np.float32)
    Y = np.empty((M, N), np.uint16)
    rc = lib().orc_tensorwise_absmax(_p(X), _p(W), M, K, N, _p(qx), _p(qw), _p(cx), _p(cw), _p(Y))
    if rc != 0:
        raise OverflowError("int8 contraction does not fit int32")
    return dict(qx=qx, qw=qw, c_x=cx[0], c_w=cw[0], Y=Y.view(np.float16))


def num_threads() -> int:
    return int(lib().orc_num_threads())


def set_num_threads(n: int) -> None:
    lib().orc_set_num_threads(int(n))
