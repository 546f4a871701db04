"""Failure detection on the GPU without a fault: a device wait that nothing
satisfies runs out after the handle's wait limit, the status word reports
it, and the handle and the CUDA context keep working."""
import pytest
import torch

import int8_quantized_matmul_outlier_b200 as m
import oracle
import workloads
from tests._parity import assert_y_close

pytestmark = pytest.mark.gpu


def test_a_wait_that_runs_out_is_reported_and_the_handle_recovers():
    p = workloads.small(64, 256, 128, 2, seed=61)
    dev = torch.device("cuda", torch.cuda.current_device())
    X = torch.from_numpy(p.X).to(dev)
    w = m.int8mm_prepare_weight(torch.from_numpy(p.W).to(dev))
    assert m.int8mm_get_status(w) == m.INT8MM_OK
    with pytest.raises(RuntimeError):
        m.int8mm_set_wait_limit(w, 999_999)   # below the 1 ms floor
    m.int8mm_set_wait_limit(w, 1_000_000)
    m.int8mm_wait_selftest(w)                  # a flag that nothing sets
    assert m.int8mm_get_status(w) == m.INT8MM_ERR_TIMEOUT
    assert m.int8mm_get_status(w) == m.INT8MM_OK  # reading the word cleared it
    m.int8mm_set_wait_limit(w, 2_000_000_000)
    y = m.int8mm_forward(w, X, p.alpha)
    assert m.int8mm_get_status(w) == m.INT8MM_OK
    r = oracle.decomp_matmul(p.X, p.W, p.alpha)
    assert_y_close(y.cpu().numpy(), r["Y"], p.X, p.W, r["idx"])
    m.int8mm_free(w)
