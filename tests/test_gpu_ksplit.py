"""The row-parallel (K-split) layer on one GPU, through the C ABI.

One process plays P ranks in turn: each rank's INT32 partial sums come from
qoq_w4a8_gemm_i32 on its slice of the packed weights (a view of the shared
INT8 activations, passed with its row stride), the partials are added (the
single-process stand-in for the NCCL all-reduce, an exact INT32 sum), and
qoq_epilogue_i32 scales them once.  The INT32 sums must equal the oracle's
bit for bit and the FP16 output must equal the single-GPU layer's bits.
Several ranks of one job are never run as separate processes on one GPU.
"""
import numpy as np
import pytest
import torch

import oracle
import w4a8_integer_gemm_b200 as q
from w4a8_integer_gemm_b200 import tp
from w4a8_integer_gemm_b200 import workloads as wl

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from w4a8_integer_gemm_b200 import build_lib
    build_lib.build()
    q.lib()


@pytest.mark.parametrize("M,K,N,G,world", [(1, 1024, 512, 128, 2), (33, 4096, 640, 128, 3), (64, 4096, 1024, 4096, 2),
                                           (200, 2048, 512, 128, 4), (17, 14336, 256, 128, 8)])
def test_ksplit_matches_single_gpu(M, K, N, G, world):
    X = wl.make_activations(M, K, wl.LLAMA, seed=900 + M)
    W = wl.make_weights(N, K, wl.LLAMA, seed=901 + N)
    packed = q.qoq_pack_weights(W.cuda(), G)
    X8, s_x = q.qoq_quant_act_per_token(X.cuda())
    acc_full = torch.zeros(M, N, dtype=torch.int32, device="cuda")
    Y_full = q.qoq_w4a8_gemm(X8, s_x, packed, acc_dbg=acc_full)
    total = torch.zeros(M, N, dtype=torch.int32, device="cuda")
    parts = []
    for (k0, k1) in tp.k_slices(K, world):
        sh = tp.shard_packed(packed, k0, k1)
        part = q.qoq_w4a8_gemm_i32(X8[:, k0:k1], sh)
        parts.append(part)
        total += part
    Y = q.qoq_epilogue_i32(total, s_x, packed.s_c)
    torch.cuda.synchronize()
    assert q.qoq_device_error() == q.QOQ_OK
    r = oracle.linear(X.numpy(), W.numpy(), G)
    assert np.array_equal(total.cpu().numpy(), r["acc"])
    assert torch.equal(total, acc_full)
    assert torch.equal(Y.view(torch.int16), Y_full.view(torch.int16))
    # each partial alone is the oracle's product on that slice
    k0, k1 = tp.k_slices(K, world)[0]
    want0 = oracle.gemm_i32(np.ascontiguousarray(r["X8"][:, k0:k1]), np.ascontiguousarray(r["W8hat"][:, k0:k1]))
    assert np.array_equal(parts[0].cpu().numpy(), want0)


@pytest.mark.parametrize("M,N", [(1, 128), (7, 512), (300, 1024)])
def test_epilogue_i32_matches_oracle(M, N):
    rng = np.random.default_rng(M + N)
    acc = rng.integers(-2 ** 28, 2 ** 28, size=(M, N), dtype=np.int64).astype(np.int32)
    s_x = (rng.random(M) * 0.05 + 1e-5).astype(np.float16).view(np.uint16)
    s_c = (rng.random(N) * 1e-3 + 1e-7).astype(np.float16).view(np.uint16)
    Y = q.qoq_epilogue_i32(torch.from_numpy(acc).cuda(), torch.from_numpy(s_x.view(np.int16)).cuda(),
                           torch.from_numpy(s_c.view(np.int16)).cuda())
    torch.cuda.synchronize()
    want = oracle.epilogue(acc, s_x, s_c)
    assert np.array_equal(Y.cpu().view(torch.int16).numpy().view(np.uint16), want)
