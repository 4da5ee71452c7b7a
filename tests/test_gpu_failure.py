"""Failure detection without a GPU fault: a bounded wait that nothing
completes must end by itself, raise the device error flag, and leave the
context usable; the next GEMM runs normally and reports no error."""
import time

import pytest
import torch

import w4a8_integer_gemm_b200 as q
from w4a8_integer_gemm_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def test_stuck_wait_times_out_and_reports():
    assert q.qoq_device_error() == q.QOQ_OK            # flag clear to begin with
    t0 = time.perf_counter()
    q.qoq_selftest_wait_timeout(2_000_000)            # 2 ms budget
    assert q.qoq_device_error() == q.QOQ_ERR_TIMEOUT  # the wait ran out and said so
    elapsed = time.perf_counter() - t0
    assert elapsed < 5.0
    assert q.qoq_device_error() == q.QOQ_OK           # reading cleared the flag

    # the context is intact: a GEMM afterwards is correct and error-free
    M, K, N = 16, 512, 512
    X = wl.make_activations(M, K, wl.LLAMA, seed=9001).cuda()
    W = wl.make_weights(N, K, wl.LLAMA, seed=9002).cuda()
    packed = q.qoq_pack_weights(W, 128)
    Y, X8, s_x = q.qoq_w4a8_linear(X, packed)
    Y2 = q.qoq_w4a8_gemm(X8, s_x, packed)
    torch.cuda.synchronize()
    assert q.qoq_device_error() == q.QOQ_OK
    assert torch.equal(Y.view(torch.int16), Y2.view(torch.int16))
