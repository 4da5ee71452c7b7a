"""The W8A8 yardstick (INT8 weights straight into the tensor cores), against
the oracle, through the C ABI: weights and scales bit-exact, INT32 sums
bit-exact, FP16 outputs within 1 ulp, over every token-tile width, ragged M
and split tiles."""
import numpy as np
import pytest
import torch

import oracle
import w4a8_integer_gemm_b200 as q
from w4a8_integer_gemm_b200 import workloads as wl

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from w4a8_integer_gemm_b200 import build_lib
    build_lib.build()
    q.lib()


def _u16(t):
    return t.cpu().view(torch.int16).numpy().view(np.uint16)


@pytest.mark.parametrize("N,K", [(128, 128), (384, 4096), (512, 24576)])
def test_quantize_w8_bit_exact(N, K):
    W = wl.make_weights(N, K, wl.QWEN, seed=40 + N)
    W[0] = 0.0
    W[1] = 1e-9
    W8, s_w = q.qoq_quantize_weights_w8(W.cuda())
    rW8, rs = oracle.quantize_weights_w8(W.numpy())
    assert np.array_equal(W8.cpu().numpy(), rW8)
    assert np.array_equal(_u16(s_w)[:N], rs)


CASES = [(1, 512, 512), (7, 1024, 384), (16, 512, 512), (33, 512, 640), (64, 4096, 1024), (100, 512, 256),
         (128, 512, 512), (200, 768, 512), (256, 512, 384), (300, 1024, 640), (513, 512, 256), (64, 8192, 8192)]


@pytest.mark.parametrize("M,K,N", CASES)
def test_w8a8_gemm_matches_oracle(M, K, N):
    X = wl.make_activations(M, K, wl.LLAMA, seed=60 + M)
    W = wl.make_weights(N, K, wl.LLAMA, seed=61 + N)
    W8, s_w = q.qoq_quantize_weights_w8(W.cuda())
    X8, s_x = q.qoq_quant_act_per_token(X.cuda())
    acc = torch.full((M, N), -5, dtype=torch.int32, device="cuda")
    Y = q.qoq_w8a8_gemm(X8, s_x, W8, s_w, acc_dbg=acc)
    torch.cuda.synchronize()
    assert q.qoq_device_error() == q.QOQ_OK
    r = oracle.linear_w8a8(X.numpy(), W.numpy())
    assert np.array_equal(acc.cpu().numpy(), r["acc"])
    g = _u16(Y).view(np.float16).astype(np.float64)
    ref = r["Y"].view(np.float16).astype(np.float64)
    ulp = np.spacing(np.abs(ref).astype(np.float16)).astype(np.float64)
    assert np.all(np.abs(g - ref) <= ulp)


def test_w8a8_repeated_calls_identical():
    X = wl.make_activations(40, 4096, wl.LLAMA, seed=70)
    W = wl.make_weights(2048, 4096, wl.LLAMA, seed=71)
    W8, s_w = q.qoq_quantize_weights_w8(W.cuda())
    X8, s_x = q.qoq_quant_act_per_token(X.cuda())
    Y0 = q.qoq_w8a8_gemm(X8, s_x, W8, s_w)
    for _ in range(5):
        assert torch.equal(q.qoq_w8a8_gemm(X8, s_x, W8, s_w).view(torch.int16), Y0.view(torch.int16))
    assert q.qoq_device_error() == q.QOQ_OK
