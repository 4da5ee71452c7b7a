"""The end-to-end calls from host memory: one call, and several pipelined on
three streams, give the bits of the device-resident layer call."""
import pytest
import torch

import w4a8_integer_gemm_b200 as q
from w4a8_integer_gemm_b200 import workloads as wl

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from w4a8_integer_gemm_b200 import build_lib
    build_lib.build()
    q.lib()


def test_host_calls_match_device_layer():
    shapes = [(1, 1024, 512), (37, 2048, 1024), (300, 1024, 2048), (5, 4096, 4096)]
    calls, refs = [], []
    for i, (M, K, N) in enumerate(shapes):
        W = wl.make_weights(N, K, wl.LLAMA, seed=6100 + i)
        layer = q.W4A8Linear(W.cuda(), group_size=128)
        X = wl.make_activations(M, K, wl.LLAMA, seed=6200 + i)
        refs.append(layer(X.cuda()).cpu())
        calls.append((X.pin_memory(), layer, torch.empty(M, N, dtype=torch.float16).pin_memory()))
    for (xh, layer, _), ref in zip(calls, refs):
        y = q.w4a8_linear_host(xh, layer)
        assert torch.equal(y.view(torch.int16), ref.view(torch.int16))
    for _ in range(3):
        for _, _, yh in calls:
            yh.fill_(float("nan"))
        outs = q.w4a8_linear_host_many(calls)
        assert q.qoq_device_error() == q.QOQ_OK
        for y, ref in zip(outs, refs):
            assert torch.equal(y.view(torch.int16), ref.view(torch.int16))


@pytest.mark.parametrize("chunk_rows", [None, 128, 1000])
def test_host_many_row_blocks(chunk_rows):
    """Calls cut into row blocks (ragged last block, and a call smaller than
    one block) return the bits of the whole device-resident layer call."""
    shapes = [(2500, 4096, 4096), (7, 1024, 512), (4500, 2048, 1024)]
    calls, refs = [], []
    for i, (M, K, N) in enumerate(shapes):
        W = wl.make_weights(N, K, wl.LLAMA, seed=6300 + i)
        layer = q.W4A8Linear(W.cuda(), group_size=128)
        X = wl.make_activations(M, K, wl.LLAMA, seed=6400 + i)
        refs.append(layer(X.cuda()).cpu())
        calls.append((X.pin_memory(), layer, torch.full((M, N), float("nan"), dtype=torch.float16).pin_memory()))
    outs = q.w4a8_linear_host_many(calls, chunk_rows=chunk_rows)
    assert q.qoq_device_error() == q.QOQ_OK
    for y, ref in zip(outs, refs):
        assert torch.equal(y.view(torch.int16), ref.view(torch.int16))
