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


# The forward's own waits: a test-only switch leaves out one kind of arrival
# (nothing else changes), the waiting side's bounded wait runs out, the
# kernels drain and exit, the status reads TIMEOUT once, and the next normal
# forward on the same handle matches the oracle.
FORWARD_WAITS = [
    # (what is left out, M, K, N, outliers, forced split K)
    ("splitk_ticket", 300, 1040, 784, 5, 2),   # prefill GEMM: a tile owner's ticket
    ("decode_ticket", 40, 2048, 4112, 5, 0),   # decode GEMM: a split n block's ticket
    ("barrier_arrival", 300, 1040, 784, 5, 0),  # single-launch activation pass: grid barrier
    ("barrier_arrival", 40, 2048, 4112, 5, 0),  # decode GEMM's own activation pass: first grid barrier
]


@pytest.mark.parametrize("what,M,K,N,n_out,split", FORWARD_WAITS)
def test_a_forward_wait_that_runs_out_is_reported_and_the_handle_recovers(what, M, K, N, n_out, split):
    bits = {"splitk_ticket": m.INT8MM_TEST_SKIP_SPLITK_TICKET,
            "decode_ticket": m.INT8MM_TEST_SKIP_DECODE_TICKET,
            "barrier_arrival": m.INT8MM_TEST_SKIP_BARRIER_ARRIVAL}[what]
    p = workloads.small(M, K, N, n_out, seed=M + K + N)
    dev = torch.device("cuda", torch.cuda.current_device())
    X = torch.from_numpy(p.X).to(dev)
    w = m.int8mm_prepare_weight(torch.from_numpy(p.W).to(dev))
    m.int8mm_set_split_k(w, split)
    m.int8mm_reserve(w, M)
    r = oracle.decomp_matmul(p.X, p.W, p.alpha)
    y = m.int8mm_forward(w, X, p.alpha)
    assert m.int8mm_get_status(w) == m.INT8MM_OK
    assert_y_close(y.cpu().numpy(), r["Y"], p.X, p.W, r["idx"])
    with pytest.raises(RuntimeError):
        m.int8mm_set_test_skip(w, 8)  # not a known arrival
    m.int8mm_set_wait_limit(w, 1_000_000)
    m.int8mm_set_test_skip(w, bits)
    m.int8mm_forward(w, X, p.alpha)
    assert m.int8mm_get_status(w) == m.INT8MM_ERR_TIMEOUT
    m.int8mm_set_test_skip(w, 0)
    m.int8mm_set_wait_limit(w, 2_000_000_000)
    for _ in range(2):
        y = m.int8mm_forward(w, X, p.alpha)
        assert m.int8mm_get_status(w) == m.INT8MM_OK
        assert_y_close(y.cpu().numpy(), r["Y"], p.X, p.W, r["idx"])
    m.int8mm_free(w)
