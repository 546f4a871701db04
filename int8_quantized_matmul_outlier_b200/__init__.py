"""Python binding of libint8mm.so, the sm_100a LLM.int8() decomposed matmul.

Argument marshalling only: every function below passes device pointers,
sizes and a CUDA stream to the C ABI declared in ``include/int8mm.h`` and
raises ``Int8mmError`` on a non-zero status.  All arithmetic runs in the
library's CUDA kernels; there is no fallback, and importing this package
fails loudly when the library has not been built.

PyTorch is used only to pass device memory and streams.
"""
from __future__ import annotations

import ctypes
import os

import torch

from . import build as _build

LIB_PATH = _build.LIB

INT8MM_OK = 0
INT8MM_ERR_INVALID_ARG = 1
INT8MM_ERR_UNSUPPORTED_SHAPE = 2
INT8MM_ERR_ALIGNMENT = 3
INT8MM_ERR_OOM = 4
INT8MM_ERR_CUDA = 5
INT8MM_ERR_TIMEOUT = 6
INT8MM_ERR_OUTLIER_CAP = 7
STATUS_NAMES = {0: "OK", 1: "INVALID_ARG", 2: "UNSUPPORTED_SHAPE", 3: "ALIGNMENT", 4: "OOM",
                5: "CUDA", 6: "TIMEOUT", 7: "OUTLIER_CAP"}
MAX_K = 65536

# Symbols of include/int8mm.h and their ctypes signatures.
_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_ST = ctypes.c_int
SIGNATURES = {
    "int8mm_prepare_weight": (_ST, [_P, _I64, _I64, _P, ctypes.POINTER(_P)]),
    "int8mm_reserve": (_ST, [_P, _I64, _P]),
    "int8mm_forward": (_ST, [_P, _P, _I64, ctypes.c_float, _P, _P]),
    "int8mm_forward_host": (_ST, [_P, _P, _I64, ctypes.c_float, _P, _P]),
    "int8mm_forward_bias": (_ST, [_P, _P, _I64, ctypes.c_float, _P, _P, _P]),
    "int8mm_forward_events": (_ST, [_P, _P, _I64, ctypes.c_float, _P, _P, ctypes.POINTER(_P)]),
    "int8mm_forward_debug": (_ST, [_P, _P, _I64, ctypes.c_float, _P, _P, _P]),
    "int8mm_get_status": (_ST, [_P]),
    "int8mm_set_wait_limit": (_ST, [_P, ctypes.c_uint64]),
    "int8mm_set_split_k": (_ST, [_P, ctypes.c_int]),
    "int8mm_wait_selftest": (_ST, [_P, _P]),
    "int8mm_set_test_skip": (_ST, [_P, ctypes.c_int]),
    "int8mm_prepare_weight_static": (_ST, [_P, _I64, _I64, _P, _I64, ctypes.c_int, _P, ctypes.POINTER(_P)]),
    "int8mm_weight_bytes": (_ST, [_P, ctypes.POINTER(ctypes.c_size_t)]),
    "int8mm_launches_per_forward": (_ST, [_P, _I64, ctypes.POINTER(ctypes.c_int)]),
    "int8mm_free": (None, [_P]),
    "int8mm_last_error": (ctypes.c_char_p, []),
    "int8mm_outlier_columns_noalloc": (_ST, [_P, _I64, _I64, ctypes.c_float, _P, _P, _P, _P]),
}


class DebugBufs(ctypes.Structure):
    """Mirror of ``int8mm_debug_bufs`` (all device pointers, NULL = skip)."""

    _fields_ = [("colmax", _P), ("outlier_idx", _P), ("outlier_count", _P), ("x_codes", _P),
                ("c_x", _P), ("w_codes_t", _P), ("c_w", _P), ("acc", _P)]


class Int8mmError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"int8mm status {status} ({STATUS_NAMES.get(status, '?')}): {message}")
        self.status = status


_lib = None


def lib() -> ctypes.CDLL:
    """Load libint8mm.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -c 'import __graft_entry__ as g; g.build()'`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def int8mm_last_error() -> str:
    return lib().int8mm_last_error().decode()


def _check(status: int) -> None:
    if status != INT8MM_OK:
        raise Int8mmError(status, int8mm_last_error())


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream if isinstance(stream, int) else stream.cuda_stream


def _dev_f16_2d(t: torch.Tensor, name: str) -> torch.Tensor:
    if not (t.is_cuda and t.dtype == torch.float16 and t.dim() == 2 and t.is_contiguous()):
        raise ValueError(f"{name} must be a contiguous 2-D float16 CUDA tensor")
    return t


class Weight:
    """A prepared weight (the library-owned handle).  Keeps a reference to
    the borrowed fp16 weight so that it outlives the handle (None for a
    static weight, which keeps what it needs itself)."""

    def __init__(self, handle: int, W: torch.Tensor | None, K: int | None = None, N: int | None = None):
        self.handle = handle
        self.W = W
        self.K, self.N = W.shape if W is not None else (K, N)

    def __del__(self):
        h, self.handle = getattr(self, "handle", None), None
        if h and _lib is not None:
            _lib.int8mm_free(h)


def int8mm_prepare_weight(W: torch.Tensor, stream=None) -> Weight:
    _dev_f16_2d(W, "W")
    K, N = W.shape
    out = _P()
    _check(lib().int8mm_prepare_weight(W.data_ptr(), K, N, _stream(stream), ctypes.byref(out)))
    return Weight(out.value, W)


def int8mm_prepare_weight_static(W: torch.Tensor, rows, max_outliers: int = 256, stream=None) -> Weight:
    """Memory-saving prepared weight: keeps the fp16 rows W[rows, :] of the
    calibrated outlier dimensions (any other outlier row is rebuilt from the
    int8 codes) and at most max_outliers (capped at K) outlier columns per
    forward.  W is not kept: it may be freed after this call."""
    _dev_f16_2d(W, "W")
    K, N = W.shape
    r = (ctypes.c_int32 * max(len(rows), 1))(*[int(x) for x in rows])
    out = _P()
    _check(lib().int8mm_prepare_weight_static(W.data_ptr(), K, N, ctypes.cast(r, _P), len(rows),
                                              int(min(max_outliers, K)), _stream(stream), ctypes.byref(out)))
    return Weight(out.value, None, K, N)


def int8mm_reserve(w: Weight, M_max: int, stream=None) -> None:
    _check(lib().int8mm_reserve(w.handle, int(M_max), _stream(stream)))


def int8mm_forward(w: Weight, X: torch.Tensor, alpha: float = 6.0, Y: torch.Tensor | None = None,
                   stream=None) -> torch.Tensor:
    _dev_f16_2d(X, "X")
    M = X.shape[0]
    if X.shape[1] != w.K:
        raise ValueError(f"X has {X.shape[1]} columns, the weight has K={w.K}")
    if Y is None:
        Y = torch.empty((M, w.N), dtype=torch.float16, device=X.device)
    _dev_f16_2d(Y, "Y")
    _check(lib().int8mm_forward(w.handle, X.data_ptr(), M, float(alpha), Y.data_ptr(), _stream(stream)))
    return Y


def int8mm_forward_bias(w: Weight, X: torch.Tensor, alpha: float = 6.0, bias: torch.Tensor | None = None,
                        Y: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """int8mm_forward plus the layer's fp16 bias [N] (None: no bias)."""
    _dev_f16_2d(X, "X")
    M = X.shape[0]
    if X.shape[1] != w.K:
        raise ValueError(f"X has {X.shape[1]} columns, the weight has K={w.K}")
    bp = None
    if bias is not None:
        if (not bias.is_cuda or bias.dtype != torch.float16 or not bias.is_contiguous()
                or bias.numel() != w.N or bias.device != X.device):
            raise ValueError("bias must be a contiguous float16 tensor of N elements on X's device")
        bp = bias.data_ptr()
    if Y is None:
        Y = torch.empty((M, w.N), dtype=torch.float16, device=X.device)
    _dev_f16_2d(Y, "Y")
    _check(lib().int8mm_forward_bias(w.handle, X.data_ptr(), M, float(alpha), bp, Y.data_ptr(), _stream(stream)))
    return Y


def int8mm_forward_host(w: Weight, X: torch.Tensor, alpha: float = 6.0, Y: torch.Tensor | None = None,
                        stream=None) -> torch.Tensor:
    """X and Y are host (CPU) float16 tensors; pin them for asynchronous copies.
    Y is valid after the stream is synchronised."""
    if X.is_cuda or X.dtype != torch.float16 or not X.is_contiguous() or X.dim() != 2:
        raise ValueError("X must be a contiguous 2-D float16 CPU tensor")
    M = X.shape[0]
    if Y is None:
        Y = torch.empty((M, w.N), dtype=torch.float16, pin_memory=X.is_pinned())
    _check(lib().int8mm_forward_host(w.handle, X.data_ptr(), M, float(alpha), Y.data_ptr(), _stream(stream)))
    return Y


def _event_handle(ev: torch.cuda.Event, stream) -> int:
    if not ev.cuda_event:
        ev.record(stream)  # torch creates the CUDA event on its first record
    return ev.cuda_event


def int8mm_forward_events(w: Weight, X: torch.Tensor, alpha: float, Y: torch.Tensor, events, stream=None):
    """Forward that records the 3 given torch.cuda.Events (timing enabled) on the
    launch stream: before the activation pass, before the GEMM, after the GEMM."""
    _dev_f16_2d(X, "X")
    _dev_f16_2d(Y, "Y")
    if len(events) != 3:
        raise ValueError("need 3 events")
    s = stream if stream is not None else torch.cuda.current_stream()
    arr = (_P * 3)(*[_event_handle(e, s) for e in events])
    _check(lib().int8mm_forward_events(w.handle, X.data_ptr(), X.shape[0], float(alpha), Y.data_ptr(),
                                       _stream(s), arr))
    return Y


def int8mm_forward_debug(w: Weight, X: torch.Tensor, alpha: float = 6.0, Y: torch.Tensor | None = None,
                         stream=None, want_acc: bool = True) -> dict:
    """Forward plus its intermediates as device tensors: colmax, outlier_idx
    (trimmed to the count), x_codes, c_x, w_codes_t, c_w and (if asked) acc."""
    _dev_f16_2d(X, "X")
    M, K = X.shape
    N = w.N
    dev = X.device
    if Y is None:
        Y = torch.empty((M, N), dtype=torch.float16, device=dev)
    out = dict(
        colmax=torch.empty(K, dtype=torch.float32, device=dev),
        outlier_idx=torch.empty(K, dtype=torch.int32, device=dev),
        outlier_count=torch.empty(1, dtype=torch.int32, device=dev),
        x_codes=torch.empty((M, K), dtype=torch.int8, device=dev),
        c_x=torch.empty(M, dtype=torch.float32, device=dev),
        w_codes_t=torch.empty((N, K), dtype=torch.int8, device=dev),
        c_w=torch.empty(N, dtype=torch.float32, device=dev),
        acc=torch.empty((M, N), dtype=torch.int32, device=dev) if want_acc else None,
    )
    d = DebugBufs(*[(t.data_ptr() if t is not None else None) for t in
                    (out["colmax"], out["outlier_idx"], out["outlier_count"], out["x_codes"],
                     out["c_x"], out["w_codes_t"], out["c_w"], out["acc"])])
    _check(lib().int8mm_forward_debug(w.handle, X.data_ptr(), M, float(alpha), Y.data_ptr(),
                                      _stream(stream), ctypes.byref(d)))
    out["Y"] = Y
    return out


def int8mm_outlier_columns_noalloc(X: torch.Tensor, alpha: float = 6.0, stream=None,
                                   want_colmax: bool = True):
    """Outlier columns of X with no device allocation inside the library:
    returns (idx [K] int32, count [1] int32, colmax [K] fp32 or None) as
    device tensors, allocated here by the caller side (PyTorch)."""
    _dev_f16_2d(X, "X")
    M, K = X.shape
    idx = torch.empty(K, dtype=torch.int32, device=X.device)
    count = torch.empty(1, dtype=torch.int32, device=X.device)
    colmax = torch.empty(K, dtype=torch.float32, device=X.device) if want_colmax else None
    _check(lib().int8mm_outlier_columns_noalloc(X.data_ptr(), M, K, float(alpha), idx.data_ptr(),
                                                count.data_ptr(),
                                                colmax.data_ptr() if colmax is not None else None,
                                                _stream(stream)))
    return idx, count, colmax


def int8mm_get_status(w: Weight) -> int:
    """Synchronises the device; returns the status code (does not raise)."""
    return int(lib().int8mm_get_status(w.handle))


def int8mm_set_wait_limit(w: Weight, timeout_ns: int) -> None:
    """Limit of each device-side wait, in ns (at least 1e6)."""
    _check(lib().int8mm_set_wait_limit(w.handle, int(timeout_ns)))


def int8mm_wait_selftest(w: Weight, stream=None) -> None:
    """Enqueue the failure-detection self-test: a device wait that runs out
    after the handle's wait limit and leaves INT8MM_ERR_TIMEOUT for
    int8mm_get_status."""
    _check(lib().int8mm_wait_selftest(w.handle, _stream(stream)))


INT8MM_TEST_SKIP_SPLITK_TICKET = 1
INT8MM_TEST_SKIP_DECODE_TICKET = 2
INT8MM_TEST_SKIP_BARRIER_ARRIVAL = 4


def int8mm_set_test_skip(w: Weight, bits: int) -> None:
    """Failure-detection tests only: later forwards leave out the arrivals
    named by `bits` (INT8MM_TEST_SKIP_*), so a device wait runs out."""
    _check(lib().int8mm_set_test_skip(w.handle, int(bits)))


def int8mm_set_split_k(w: Weight, split: int) -> None:
    """Pieces along K per prefill GEMM tile: 0 automatic, 1..4 forced."""
    _check(lib().int8mm_set_split_k(w.handle, int(split)))


def int8mm_weight_bytes(w: Weight) -> int:
    n = ctypes.c_size_t()
    _check(lib().int8mm_weight_bytes(w.handle, ctypes.byref(n)))
    return int(n.value)


def int8mm_launches_per_forward(w: Weight, M: int) -> int:
    n = ctypes.c_int()
    _check(lib().int8mm_launches_per_forward(w.handle, int(M), ctypes.byref(n)))
    return int(n.value)


def int8mm_free(w: Weight) -> None:
    h, w.handle = w.handle, None
    if h:
        lib().int8mm_free(h)


from .linear import Linear8bitLt  # noqa: E402  (the layer over the functions above)
