"""The outlier-detection entry point that allocates no device memory.

It exists for callers that cannot allocate device memory where they need the
outlier set (an engine plugin's enqueue step, a serving loop that forbids
allocation after warm-up, a process whose caching allocator holds nearly all
of the memory).  Its scratch is a static 1 MiB device array shared by every
call.  These tests check it, through the C ABI, against the outlier set,
count and column maxima that the allocating forward reports and against the
CPU oracle, on two calls in a row (so the second call runs on scratch the
first one left behind), and check that a call takes no device memory.
This file is named to be collected last.
"""
import ctypes

import numpy as np
import pytest
import torch

import int8_quantized_matmul_outlier_b200 as m
import oracle
import workloads

pytestmark = pytest.mark.gpu


def reference_outliers(X, W):
    w = m.int8mm_prepare_weight(W)
    d = m.int8mm_forward_debug(w, X, 6.0, want_acc=False)
    torch.cuda.synchronize()
    cnt = int(d["outlier_count"].item())
    out = (d["outlier_idx"][:cnt].cpu().numpy(), cnt, d["colmax"].cpu().numpy())
    m.int8mm_free(w)
    return out


def test_noalloc_matches_forward_on_two_calls_in_a_row():
    dev = torch.device("cuda", torch.cuda.current_device())
    problems = [workloads.small(300, 1040, 64, 5, seed=901), workloads.opt13b_prefill(with_weight=False)]
    problems[1].W = workloads.weight(5120, 16, 902)
    for p in problems:
        X = torch.from_numpy(p.X).to(dev)
        W = torch.from_numpy(p.W).to(dev)
        ref_idx, ref_cnt, ref_colmax = reference_outliers(X, W)
        orc_colmax, orc_idx = oracle.outlier_columns(p.X, 6.0)
        for _ in range(2):
            idx, cnt, colmax = m.int8mm_outlier_columns_noalloc(X, 6.0)
            torch.cuda.synchronize()
            n = int(cnt.item())
            assert n == ref_cnt == orc_idx.size == p.planted.size
            assert np.array_equal(idx[:n].cpu().numpy(), ref_idx)
            assert np.array_equal(idx[:n].cpu().numpy(), orc_idx)
            assert np.array_equal(colmax.cpu().numpy(), ref_colmax)
            assert np.array_equal(colmax.cpu().numpy(), orc_colmax)


def test_noalloc_call_takes_no_device_memory():
    # outputs allocated up front; after one warm-up call (which loads the
    # kernel and looks up the static array), further calls through the C ABI
    # must leave the device's free memory unchanged
    dev = torch.device("cuda", torch.cuda.current_device())
    p = workloads.small(2000, 4096, 16, 7, seed=903)
    X = torch.from_numpy(p.X).to(dev)
    M, K = p.X.shape
    idx = torch.empty(K, dtype=torch.int32, device=dev)
    cnt = torch.empty(1, dtype=torch.int32, device=dev)
    colmax = torch.empty(K, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream().cuda_stream

    def call():
        return m.lib().int8mm_outlier_columns_noalloc(X.data_ptr(), M, K, ctypes.c_float(6.0), idx.data_ptr(),
                                                      cnt.data_ptr(), colmax.data_ptr(), stream)

    assert call() == m.INT8MM_OK
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    for _ in range(3):
        assert call() == m.INT8MM_OK
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0
    orc_colmax, orc_idx = oracle.outlier_columns(p.X, 6.0)
    n = int(cnt.item())
    assert n == orc_idx.size == 7
    assert np.array_equal(idx[:n].cpu().numpy(), orc_idx)
    assert np.array_equal(colmax.cpu().numpy(), orc_colmax)


def test_noalloc_no_rows():
    # M == 0: no outlier columns, and the maximum over no rows is 0
    dev = torch.device("cuda", torch.cuda.current_device())
    X = torch.zeros((0, 64), dtype=torch.float16, device=dev)
    idx, cnt, colmax = m.int8mm_outlier_columns_noalloc(X, 6.0)
    torch.cuda.synchronize()
    assert int(cnt.item()) == 0
    assert (colmax == 0).all()


def test_noalloc_rejects_sizes_beyond_its_scratch():
    dev = torch.device("cuda", torch.cuda.current_device())
    K = m.MAX_K + 16
    X = torch.zeros((1, K), dtype=torch.float16, device=dev)
    with pytest.raises(m.Int8mmError) as e:
        m.int8mm_outlier_columns_noalloc(X, 6.0)
    assert e.value.status == m.INT8MM_ERR_UNSUPPORTED_SHAPE
    assert "no-allocation" in str(e.value)
