"""The activation quantizer and the GEMM captured in one CUDA graph.

A decode step replays the same launches many times; the kernels must give
the same bits when they run from a graph (programmatic dependent launch
edges between them) as when they are launched one by one, and the split-tile
counters in the workspace must be left ready for the next replay.  The
outputs are also checked against the oracle on a sample.
"""
import numpy as np
import pytest
import torch

import oracle
import w4a8_integer_gemm_b200 as q
from w4a8_integer_gemm_b200 import workloads as wl

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("M,K,N,G", [(1, 4096, 14336, 128), (64, 4096, 14336, 4096), (200, 1024, 2048, 128)])
def test_graph_replay_matches_eager(M, K, N, G):
    q.qoq_set_gemm_a_in_tmem(True)
    X = wl.make_activations(M, K, wl.LLAMA, seed=4100 + M)
    W = wl.make_weights(N, K, wl.LLAMA, seed=4200 + M)
    dev = torch.device("cuda")
    packed = q.qoq_pack_weights(W.to(dev), G)
    Xd = X.to(dev)
    # two layers in a row, as in a decode step, each with its own buffers
    bufs = []
    for _ in range(2):
        X8 = torch.empty(M, K, dtype=torch.int8, device=dev)
        s_x = torch.empty(max(M, 8), dtype=torch.int16, device=dev)
        Y = torch.empty(M, N, dtype=torch.float16, device=dev)
        ws = torch.zeros(q.qoq_gemm_workspace_bytes(M, N, K, G), dtype=torch.uint8, device=dev)
        bufs.append((X8, s_x, Y, ws))

    def step(st):
        for X8, s_x, Y, ws in bufs:
            q.qoq_quant_act_per_token(Xd, X8, s_x, stream=st)
            q.qoq_w4a8_gemm(X8, s_x, packed, Y=Y, workspace=ws, stream=st)

    main = torch.cuda.current_stream()
    step(main)
    torch.cuda.synchronize()
    assert q.qoq_device_error() == q.QOQ_OK
    eager = [b[2].clone() for b in bufs]
    for b in bufs:
        b[2].fill_(0)

    cap = torch.cuda.Stream()
    cap.wait_stream(main)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=cap):
        step(cap)
    main.wait_stream(cap)
    for rep in range(3):
        for b in bufs:
            b[2].fill_(0)
        g.replay()
        torch.cuda.synchronize()
        assert q.qoq_device_error() == q.QOQ_OK
        for b, e in zip(bufs, eager):
            assert torch.equal(b[2].view(torch.int16), e.view(torch.int16)), f"replay {rep} differs"
        # the counters at the head of each workspace are back at zero
        for b in bufs:
            assert int(b[3][:8192].view(torch.int32).abs().sum()) == 0
    del g

    rng = np.random.default_rng(M)
    rows = np.unique(np.concatenate([rng.choice(M, size=min(M, 8), replace=False), [0, M - 1]]))
    cols = np.unique(np.concatenate([rng.choice(N, size=32, replace=False), [0, N - 1]]))
    r = oracle.linear_sampled(X.numpy(), W.numpy(), G, rows, cols)
    got = eager[1][torch.as_tensor(rows)][:, torch.as_tensor(cols)].cpu().view(torch.int16).numpy().view(np.uint16)
    gf = got.view(np.float16).astype(np.float64)
    rf = r["Y"].view(np.float16).astype(np.float64)
    ulp = np.spacing(np.abs(rf).astype(np.float16)).astype(np.float64)
    assert np.all(np.abs(gf - rf) <= ulp)
