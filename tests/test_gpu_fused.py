"""The layer call (qoq_w4a8_linear), as two kernels (default) and as one
GEMM launch that quantizes its own rows: each must give exactly what the
two separate calls give -- X8, s_x and Y bit for bit -- on every output,
over repeated calls (the one-launch form resets its own counters) and from
a CUDA graph; a sample is also checked against the oracle."""
import numpy as np
import pytest
import torch

import oracle
import w4a8_integer_gemm_b200 as q
from w4a8_integer_gemm_b200 import workloads as wl

pytestmark = pytest.mark.gpu

SHAPES = [
    # M, K, N, G: decode widths, several rows per quantizing warp (M > 4 x 148),
    # a long row (K = 24576), 256-token tiles
    (1, 4096, 14336, 128),
    (33, 4096, 14336, 4096),
    (64, 4096, 14336, 128),
    (200, 1024, 2048, 128),
    (1000, 512, 512, 128),
    (5, 24576, 256, 128),
    (700, 2048, 1024, 2048),
]


@pytest.fixture(params=[False, True], ids=["two_kernels", "one_launch"])
def in_kernel(request):
    q.qoq_set_linear_in_kernel_quant(request.param)
    yield request.param
    q.qoq_set_linear_in_kernel_quant(False)


@pytest.mark.parametrize("M,K,N,G", SHAPES, ids=[f"M{m}_K{k}_N{n}_G{g}" for m, k, n, g in SHAPES])
def test_fused_equals_separate(M, K, N, G, in_kernel):
    q.qoq_set_gemm_a_in_tmem(True)
    dev = torch.device("cuda")
    X = wl.make_activations(M, K, wl.LLAMA, seed=6100 + M)
    W = wl.make_weights(N, K, wl.LLAMA, seed=6200 + M)
    packed = q.qoq_pack_weights(W.to(dev), G)
    Xd = X.to(dev)
    X8r, sxr = q.qoq_quant_act_per_token(Xd)
    Yr = q.qoq_w4a8_gemm(X8r, sxr, packed)
    ws = torch.zeros(q.qoq_gemm_workspace_bytes(M, N, K, G), dtype=torch.uint8, device=dev)
    X8 = torch.empty(M, K, dtype=torch.int8, device=dev)
    sx = torch.empty(max(M, 8), dtype=torch.int16, device=dev)
    Y = torch.empty(M, N, dtype=torch.float16, device=dev)
    for run in range(3):
        X8.fill_(0)
        sx.fill_(0)
        Y.fill_(0)
        q.qoq_w4a8_linear(Xd, packed, X8=X8, s_x=sx, Y=Y, workspace=ws)
        torch.cuda.synchronize()
        assert q.qoq_device_error() == q.QOQ_OK
        assert torch.equal(X8, X8r), f"run {run}: X8 differs"
        assert torch.equal(sx[:M], sxr[:M]), f"run {run}: s_x differs"
        assert torch.equal(Y.view(torch.int16), Yr.view(torch.int16)), f"run {run}: Y differs"
        assert int(ws[:8192].view(torch.int32).abs().sum()) == 0

    main = torch.cuda.current_stream()
    cap = torch.cuda.Stream()
    cap.wait_stream(main)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=cap):
        q.qoq_w4a8_linear(Xd, packed, X8=X8, s_x=sx, Y=Y, workspace=ws, stream=cap)
    main.wait_stream(cap)
    for run in range(3):
        Y.fill_(0)
        g.replay()
        torch.cuda.synchronize()
        assert q.qoq_device_error() == q.QOQ_OK
        assert torch.equal(Y.view(torch.int16), Yr.view(torch.int16)), f"replay {run}: Y differs"
    del g

    rng = np.random.default_rng(M + K)
    rows = np.unique(np.concatenate([rng.choice(M, size=min(M, 6), replace=False), [0, M - 1]]))
    cols = np.unique(np.concatenate([rng.choice(N, size=min(N, 24), replace=False), [0, N - 1]]))
    r = oracle.linear_sampled(X.numpy(), W.numpy(), G, rows, cols)
    got = Y[torch.as_tensor(rows)][:, torch.as_tensor(cols)].cpu().view(torch.int16).numpy().view(np.uint16)
    gf = got.view(np.float16).astype(np.float64)
    rf = r["Y"].view(np.float16).astype(np.float64)
    ulp = np.spacing(np.abs(rf).astype(np.float16)).astype(np.float64)
    assert np.all(np.abs(gf - rf) <= ulp)
