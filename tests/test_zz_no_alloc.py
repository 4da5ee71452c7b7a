"""The allocation-free GEMM entry point, checked against the regular one.

qoq_w4a8_gemm_noalloc exists for callers that cannot allocate while they run
the layer: an inference engine's execute step where allocating is forbidden
or would synchronize the device, a plug-in with no allocator, a real-time
path.  It keeps the GEMM's scratch in a fixed buffer inside the library.
This test calls it through the C ABI twice in a row (the second call finds
the first call's leftovers in the shared buffer) and compares its FP16
output with qoq_w4a8_gemm's, to the 1-ulp bar the other parity tests use.
It needs nothing from earlier tests, so it passes alone in a fresh process
as well as after the rest of the suite (this file is collected last).
"""
import ctypes

import numpy as np
import pytest
import torch

import w4a8_integer_gemm_b200 as q
from w4a8_integer_gemm_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def _half_bits(t):
    return t.cpu().view(torch.int16).numpy().view(np.uint16)


def _within_1ulp(a_bits, b_bits):
    a = a_bits.view(np.float16).astype(np.float64)
    b = b_bits.view(np.float16).astype(np.float64)
    ulp = np.spacing(np.abs(b).astype(np.float16)).astype(np.float64)
    return bool(np.all(np.abs(a - b) <= ulp))


@pytest.mark.parametrize("M,K,N,G", [(1, 4096, 2048, 128), (16, 1024, 1536, 1024), (64, 4096, 1024, 128),
                                     (33, 512, 640, 128)])
def test_noalloc_matches_regular_entry(M, K, N, G):
    from w4a8_integer_gemm_b200 import build_lib
    build_lib.build()
    L = q.lib()
    X = wl.make_activations(M, K, wl.LLAMA, seed=900 + M).cuda()
    W = wl.make_weights(N, K, wl.LLAMA, seed=901 + N).cuda()
    packed = q.qoq_pack_weights(W, G)
    X8, s_x = q.qoq_quant_act_per_token(X)
    ref = q.qoq_w4a8_gemm(X8, s_x, packed)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    outs = []
    for _ in range(2):
        Y = torch.full((M, N), float("nan"), dtype=torch.float16, device="cuda")
        st = L.qoq_w4a8_gemm_noalloc(ctypes.c_void_p(X8.data_ptr()), ctypes.c_void_p(s_x.data_ptr()),
                                     ctypes.c_void_p(packed.Wp.data_ptr()), ctypes.c_void_p(packed.s_c.data_ptr()),
                                     ctypes.c_void_p(packed.s_g.data_ptr()), ctypes.c_void_p(packed.zs.data_ptr()),
                                     M, N, K, G, ctypes.c_void_p(Y.data_ptr()), stream)
        assert st == q.QOQ_OK, q.qoq_status_string(st)
        outs.append(Y)
    torch.cuda.synchronize()
    assert q.qoq_device_error() == q.QOQ_OK
    r = _half_bits(ref)
    for Y in outs:
        assert _within_1ulp(_half_bits(Y), r)


def test_noalloc_rejects_oversized_shape():
    L = q.lib()
    # 4096 tokens need far more split-tile scratch than the built-in buffer
    assert q.qoq_gemm_workspace_bytes(4096, 8192, 8192, 128) > q.QOQ_NOALLOC_SCRATCH_BYTES
    fake = ctypes.c_void_p(1 << 20)   # never dereferenced: the size check comes first
    st = L.qoq_w4a8_gemm_noalloc(fake, fake, fake, fake, fake, fake, 4096, 8192, 8192, 128, fake, None)
    assert st == q.QOQ_ERR_SCRATCH_TOO_SMALL
