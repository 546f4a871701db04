"""The C ABI on the host: the library loads, exports every symbol that
include/int8mm.h declares, and rejects bad arguments before touching a GPU."""
import ctypes
import os
import re

import pytest

import int8_quantized_matmul_outlier_b200 as m

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "int8mm.h")


def declared_functions():
    text = open(HEADER, encoding="utf-8").read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(int8mm_[a-z_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("int8mm_prepare_weight", "int8mm_forward", "int8mm_free"):
        assert required in names
    assert set(names) == set(m.SIGNATURES), set(names) ^ set(m.SIGNATURES)


def test_library_exports_every_declared_symbol():
    L = ctypes.CDLL(m.LIB_PATH)
    for name in declared_functions():
        assert hasattr(L, name), name


def test_prepare_rejects_bad_arguments_on_the_host():
    L = m.lib()
    out = ctypes.c_void_p(1234)
    assert L.int8mm_prepare_weight(None, 64, 64, None, ctypes.byref(out)) == m.INT8MM_ERR_INVALID_ARG
    assert out.value is None
    assert "NULL" in m.int8mm_last_error()
    assert L.int8mm_prepare_weight(None, 64, 64, None, None) == m.INT8MM_ERR_INVALID_ARG
    fake = ctypes.c_void_p(4096)  # never dereferenced: shape checks come first
    for K, N in ((15, 64), (64, 8), (0, 64), (64, 20), (m.MAX_K + 16, 64)):
        assert L.int8mm_prepare_weight(fake, K, N, None, ctypes.byref(out)) == m.INT8MM_ERR_UNSUPPORTED_SHAPE
    assert L.int8mm_prepare_weight(ctypes.c_void_p(4098), 64, 64, None, ctypes.byref(out)) == \
        m.INT8MM_ERR_ALIGNMENT


def test_static_prepare_rejects_bad_rows_on_the_host():
    L = m.lib()
    out = ctypes.c_void_p(1234)
    fake = ctypes.c_void_p(4096)  # never dereferenced: the row checks come first

    def rows(*v):
        return ctypes.cast((ctypes.c_int32 * len(v))(*v), ctypes.c_void_p)

    cases = [(None, 1, 4),            # rows missing
             (rows(1, 2), -1, 4),     # negative count
             (rows(3, 3), 2, 4),      # repeated dimension
             (rows(64), 1, 4),        # outside [0, K)
             (rows(-1), 1, 4),
             (rows(1), 1, 0),         # no room for outliers
             (rows(1), 1, 65)]        # more room than K
    for r, n, cap in cases:
        st = L.int8mm_prepare_weight_static(fake, 64, 64, r, n, cap, None, ctypes.byref(out))
        assert st == m.INT8MM_ERR_INVALID_ARG, (n, cap)
        assert out.value is None
    assert L.int8mm_prepare_weight_static(fake, 15, 64, None, 0, 4, None, ctypes.byref(out)) == \
        m.INT8MM_ERR_UNSUPPORTED_SHAPE


def test_calls_on_an_unknown_handle_are_rejected():
    L = m.lib()
    bogus = ctypes.c_void_p(0xdead0)
    assert L.int8mm_forward(bogus, None, 4, 6.0, None, None) == m.INT8MM_ERR_INVALID_ARG
    assert "handle" in m.int8mm_last_error()
    assert L.int8mm_forward_host(bogus, None, 4, 6.0, None, None) == m.INT8MM_ERR_INVALID_ARG
    assert L.int8mm_forward_debug(bogus, None, 4, 6.0, None, None, None) == m.INT8MM_ERR_INVALID_ARG
    assert L.int8mm_get_status(bogus) == m.INT8MM_ERR_INVALID_ARG
    assert L.int8mm_reserve(bogus, 16, None) == m.INT8MM_ERR_INVALID_ARG
    assert L.int8mm_set_wait_limit(bogus, 1000) == m.INT8MM_ERR_INVALID_ARG
    assert L.int8mm_set_split_k(bogus, 2) == m.INT8MM_ERR_INVALID_ARG
    assert L.int8mm_wait_selftest(bogus, None) == m.INT8MM_ERR_INVALID_ARG
    n = ctypes.c_size_t()
    assert L.int8mm_weight_bytes(bogus, ctypes.byref(n)) == m.INT8MM_ERR_INVALID_ARG
    L.int8mm_free(None)    # no-op
    L.int8mm_free(bogus)   # unknown handle: no-op


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(m, "_lib", None)
    monkeypatch.setattr(m, "LIB_PATH", str(tmp_path / "absent.so"))
    with pytest.raises(RuntimeError, match="missing"):
        m.lib()
