"""The decode kernel for M <= 8 tokens against the oracle and against the
tensor-core GEMM, through the C ABI.

Both kernels compute the same INT32 sums (exact in any order) and round the
output through the same epilogue, so every case is bit-identical between
them; the oracle pins both.  Cases span 1-8 tokens (and 9-16, which take
the GEMM whatever the switch says), K split over clusters of 1, 2 and 4
CTAs (by N), an N above the decode kernel's limit (the GEMM), both table layouts
(128-wide groups, per channel), K from one block to 64 blocks (fewer blocks
than the CTA's warps, and several per warp), N from one CTA of 32 channels
up, back-to-back launches on one stream and in a CUDA graph.
"""
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
    yield
    q.qoq_set_gemm_gemv(True)


def _u16(t):
    return t.cpu().view(torch.int16).numpy().view(np.uint16)


CASES = [(1, 128, 128, 128), (1, 512, 384, 512), (2, 1024, 256, 128), (3, 4096, 640, 128),
         (4, 2048, 1024, 2048), (5, 8192, 512, 128), (7, 1536, 128, 1536), (8, 4096, 2048, 128),
         (8, 8192, 256, 8192), (9, 1024, 384, 128), (12, 2048, 128, 2048), (16, 4096, 1024, 128),
         (16, 8192, 512, 8192), (3, 2048, 4096, 128), (6, 14336, 4096, 128), (2, 4096, 8192, 128),
         (4, 1024, 20480, 128)]


@pytest.mark.parametrize("M,K,N,G", CASES)
def test_gemv_matches_oracle_and_gemm(M, K, N, G):
    X = wl.make_activations(M, K, wl.LLAMA, seed=4200 + M + K)
    W = wl.make_weights(N, K, wl.LLAMA, seed=4300 + N + K)
    packed = q.qoq_pack_weights(W.cuda(), G)
    X8, s_x = q.qoq_quant_act_per_token(X.cuda())
    out = {}
    try:
        for gemv in (True, False):
            q.qoq_set_gemm_gemv(gemv)
            acc = torch.full((M, N), -7, dtype=torch.int32, device="cuda")
            Y = q.qoq_w4a8_gemm(X8, s_x, packed, acc_dbg=acc)
            torch.cuda.synchronize()
            assert q.qoq_device_error() == q.QOQ_OK
            out[gemv] = (acc.cpu().numpy(), _u16(Y))
    finally:
        q.qoq_set_gemm_gemv(True)
    r = oracle.linear(X.numpy(), W.numpy(), G)
    assert np.array_equal(out[True][0], r["acc"])
    assert np.array_equal(out[True][0], out[False][0])
    assert np.array_equal(out[True][1], out[False][1])
    got = out[True][1].view(np.float16).astype(np.float64)
    ref = r["Y"].view(np.float16).astype(np.float64)
    ulp = np.spacing(np.abs(ref).astype(np.float16)).astype(np.float64)
    assert not (np.abs(got - ref) > ulp).any()


def test_gemv_chain_and_graph_identical():
    """Eight launches back to back (each may start while the previous one
    runs) and the same eight replayed from a CUDA graph give the bits of a
    single launch."""
    M, K, N, G = 6, 4096, 1024, 128
    X = wl.make_activations(M, K, wl.LLAMA, seed=4400)
    W = wl.make_weights(N, K, wl.LLAMA, seed=4401)
    packed = q.qoq_pack_weights(W.cuda(), G)
    X8, s_x = q.qoq_quant_act_per_token(X.cuda())
    ref = q.qoq_w4a8_gemm(X8, s_x, packed)
    ws = torch.zeros(q.qoq_gemm_workspace_bytes(M, N, K, G), dtype=torch.uint8, device="cuda")
    Ys = [torch.empty(M, N, dtype=torch.float16, device="cuda") for _ in range(8)]
    for Yi in Ys:
        q.qoq_w4a8_gemm(X8, s_x, packed, Y=Yi, workspace=ws)
    torch.cuda.synchronize()
    for Yi in Ys:
        assert torch.equal(Yi.view(torch.int16), ref.view(torch.int16))
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        for Yi in Ys:
            q.qoq_w4a8_gemm(X8, s_x, packed, Y=Yi, workspace=ws, stream=s)
    torch.cuda.current_stream().wait_stream(s)
    for Yi in Ys:
        Yi.fill_(0)
    g.replay()
    torch.cuda.synchronize()
    assert q.qoq_device_error() == q.QOQ_OK
    for Yi in Ys:
        assert torch.equal(Yi.view(torch.int16), ref.view(torch.int16))
    del g
