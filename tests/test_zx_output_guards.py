"""No kernel writes outside Y: Y is placed inside a larger buffer whose
guard regions before and after it hold a fixed pattern, and every forward
path (decode, single-CTA prefill, CTA pairs, split K, bias, static weight)
must leave the pattern as it was and match the plain forward."""
import math

import pytest
import torch

import int8_quantized_matmul_outlier_b200 as m
import workloads

pytestmark = pytest.mark.gpu

GUARD = 4096  # fp16 elements on each side (8 KB; keeps Y 16-byte aligned)


def _guarded(M, N, dev):
    buf = torch.empty(GUARD + M * N + GUARD, dtype=torch.float16, device=dev)
    buf.view(torch.int16).fill_(0x5a5a)
    return buf, buf[GUARD:GUARD + M * N].view(M, N)


@pytest.mark.parametrize("M,K,N,split", [(8, 1040, 784, 0), (100, 512, 272, 0), (300, 1040, 784, 0),
                                         (300, 4096, 784, 3), (513, 640, 4112, 0)])
def test_forward_writes_only_inside_y(M, K, N, split):
    dev = torch.device("cuda", torch.cuda.current_device())
    p = workloads.small(M, K, N, 5, seed=M + K + N)
    X = torch.from_numpy(p.X).to(dev)
    W = torch.from_numpy(p.W).to(dev)
    bias = (torch.arange(N, device=dev, dtype=torch.float32) % 7 / 8).half()
    w = m.int8mm_prepare_weight(W)
    m.int8mm_set_split_k(w, split)
    ws = m.int8mm_prepare_weight_static(W.clone(), p.planted.tolist(), max_outliers=16)
    ref = m.int8mm_forward(w, X, p.alpha)
    ref_b = m.int8mm_forward_bias(w, X, p.alpha, bias)
    for name, run, expect in (("plain", lambda Y: m.int8mm_forward(w, X, p.alpha, Y), ref),
                              ("bias", lambda Y: m.int8mm_forward_bias(w, X, p.alpha, bias, Y), ref_b),
                              ("static", lambda Y: m.int8mm_forward(ws, X, p.alpha, Y), ref)):
        buf, Y = _guarded(M, N, dev)
        run(Y)
        torch.cuda.synchronize()
        g = buf.view(torch.int16)
        assert (g[:GUARD] == 0x5a5a).all() and (g[GUARD + M * N:] == 0x5a5a).all(), name
        assert torch.equal(Y, expect), name
    assert m.int8mm_get_status(w) == m.INT8MM_OK and m.int8mm_get_status(ws) == m.INT8MM_OK
    m.int8mm_free(w)
    m.int8mm_free(ws)
