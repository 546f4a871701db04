"""The outlier-detection entry point that allocates no device memory.

It exists for callers that cannot allocate device memory where they need the
outlier set (an engine plugin's enqueue step, a serving loop that forbids
allocation after warm-up, a process whose caching allocator holds nearly all
of the memory).  Its scratch is a static 1 MiB device array shared by every
call.  These tests check it, through the C ABI, against the outlier set,
count and column maxima that the allocating forward reports, on two calls in
a row (so the second call runs on scratch the first one left behind).
This file is named to be collected last.
"""
import numpy as np
import pytest
import torch

import int8_quantized_matmul_outlier_b200 as m
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
        for _ in range(2):
            idx, cnt, colmax = m.int8mm_outlier_columns_noalloc(X, 6.0)
            torch.cuda.synchronize()
            n = int(cnt.item())
            assert n == ref_cnt == p.planted.size
            assert np.array_equal(idx[:n].cpu().numpy(), ref_idx)
            assert np.array_equal(colmax.cpu().numpy(), ref_colmax)


def test_noalloc_rejects_sizes_beyond_its_scratch():
    dev = torch.device("cuda", torch.cuda.current_device())
    K = m.MAX_K + 16
    X = torch.zeros((1, K), dtype=torch.float16, device=dev)
    with pytest.raises(m.Int8mmError) as e:
        m.int8mm_outlier_columns_noalloc(X, 6.0)
    assert e.value.status == m.INT8MM_ERR_UNSUPPORTED_SHAPE
    assert "no-allocation" in str(e.value)
