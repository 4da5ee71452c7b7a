"""Output-side fusion in the GEMM epilogue, against the oracle, through the C ABI.

Residual add: bit-exact with the oracle's FP16 add after the layer.
SiLU-gated pair: within 1 FP16 ulp of the oracle (binary64 silu and product,
rounded once; the kernel evaluates silu in FP32 with IEEE division).
Shapes span the token-tile widths (16 ... 256), ragged M, split tiles and
both group sizes; the full-size Llama-3-8B gate/up shape is checked on
sampled outputs.
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


def _u16(t):
    return t.cpu().view(torch.int16).numpy().view(np.uint16)


def _within_1ulp(got_bits, ref_bits):
    g = got_bits.view(np.float16).astype(np.float64)
    r = ref_bits.view(np.float16).astype(np.float64)
    ulp = np.spacing(np.abs(r).astype(np.float16)).astype(np.float64)
    bad = ~((np.abs(g - r) <= ulp) | (np.isinf(g) & np.isinf(r) & (np.sign(g) == np.sign(r))))
    return int(bad.sum())


CASES = [(1, 512, 512, 128), (16, 1024, 384, 1024), (33, 512, 640, 128), (64, 4096, 1024, 128),
         (100, 512, 256, 128), (200, 768, 512, 128), (300, 1024, 640, 128), (513, 512, 256, 512)]


@pytest.mark.parametrize("M,K,N,G", CASES)
@pytest.mark.parametrize("alias", [False, True])
def test_residual_bit_exact(M, K, N, G, alias):
    X = wl.make_activations(M, K, wl.LLAMA, seed=500 + M)
    W = wl.make_weights(N, K, wl.LLAMA, seed=501 + N)
    R = (torch.randn(M, N, generator=torch.Generator().manual_seed(502 + M)) * 3).half()
    packed = q.qoq_pack_weights(W.cuda(), G)
    X8, s_x = q.qoq_quant_act_per_token(X.cuda())
    Rd = R.cuda()
    Y = Rd if alias else torch.full((M, N), float("nan"), dtype=torch.float16, device="cuda")
    q.qoq_w4a8_gemm_fused(X8, s_x, packed, q.QOQ_EPILOGUE_RESIDUAL, residual=Rd, Y=Y)
    torch.cuda.synchronize()
    assert q.qoq_device_error() == q.QOQ_OK
    ref = oracle.linear(X.numpy(), W.numpy(), G)
    want = oracle.epilogue_residual(ref["acc"], ref["s_x"], ref["s_c"], R.numpy())
    assert np.array_equal(_u16(Y), want)


@pytest.mark.parametrize("M,K,N,G", CASES)
def test_plain_kind_equals_gemm(M, K, N, G):
    X = wl.make_activations(M, K, wl.LLAMA, seed=510 + M)
    W = wl.make_weights(N, K, wl.LLAMA, seed=511 + N)
    packed = q.qoq_pack_weights(W.cuda(), G)
    X8, s_x = q.qoq_quant_act_per_token(X.cuda())
    Y0 = q.qoq_w4a8_gemm(X8, s_x, packed)
    Y1 = q.qoq_w4a8_gemm_fused(X8, s_x, packed, q.QOQ_EPILOGUE_NONE)
    torch.cuda.synchronize()
    assert torch.equal(Y0.view(torch.int16), Y1.view(torch.int16))


def _gate_up_case(M, K, N, G, seed):
    X = wl.make_activations(M, K, wl.LLAMA, seed=seed)
    W = wl.make_weights(N, K, wl.LLAMA, seed=seed + 1)
    packed = q.qoq_pack_weights_gate_up(W.cuda(), G)
    X8, s_x = q.qoq_quant_act_per_token(X.cuda())
    Y = q.qoq_w4a8_gemm_fused(X8, s_x, packed, q.QOQ_EPILOGUE_SILU_MUL)
    torch.cuda.synchronize()
    assert q.qoq_device_error() == q.QOQ_OK
    return X, W, packed, Y


def _packed_row_of(N):
    """Packed row of each natural row of a gate/up pair (the header's layout)."""
    I = N // 2
    nat = np.empty(N, np.int64)
    for p in range(N // 128):
        for r in range(128):
            nat[128 * p + r] = 64 * p + r if r < 64 else I + 64 * p + r - 64
    pos = np.empty(N, np.int64)
    pos[nat] = np.arange(N)
    return pos


@pytest.mark.parametrize("M,K,N,G", CASES)
def test_silu_mul_within_1ulp(M, K, N, G):
    X, W, packed, Y = _gate_up_case(M, K, N, G, seed=520 + M)
    ref = oracle.linear(X.numpy(), W.numpy(), G)
    want = oracle.epilogue_silu_mul(ref["acc"], ref["s_x"], ref["s_c"])
    assert Y.shape == (M, N // 2)
    assert _within_1ulp(_u16(Y), want) == 0
    # the channel scales sit at the packed positions the header states
    pos = _packed_row_of(N)
    assert np.array_equal(_u16(packed.s_c)[pos], ref["s_c"])


@pytest.mark.parametrize("M", [64, 1024])
def test_silu_mul_llama_gate_up_sampled(M):
    """Full-size Llama-3-8B gate/up (K = 4096, N = 2 x 14336), sampled outputs."""
    K, N, G = 4096, 28672, 128
    X, W, packed, Y = _gate_up_case(M, K, N, G, seed=530 + M)
    I = N // 2
    rng = np.random.default_rng(M)
    rows = np.unique(np.concatenate([[0, M - 1], rng.integers(0, M, 14)]))
    cols = np.unique(np.concatenate([[0, I - 1, 63, 64], rng.integers(0, I, 60)]))
    ref = oracle.linear_sampled(X.numpy(), W.numpy(), G, rows, np.concatenate([cols, I + cols]))
    want = oracle.epilogue_silu_mul(ref["acc"], ref["s_x"], ref["s_c"])
    got = _u16(Y)[np.ix_(rows, cols)]
    assert _within_1ulp(got, want) == 0


def test_fused_rejects_bad_arguments():
    W = wl.make_weights(256, 512, wl.LLAMA, seed=1).cuda()
    packed = q.qoq_pack_weights(W, 128)
    X8, s_x = q.qoq_quant_act_per_token(wl.make_activations(4, 512, wl.LLAMA, 2).cuda())
    with pytest.raises(ValueError):
        q.qoq_w4a8_gemm_fused(X8, s_x, packed, q.QOQ_EPILOGUE_SILU_MUL)   # not gate/up packed
    with pytest.raises(q.QoQError):
        q.qoq_w4a8_gemm_fused(X8, s_x, packed, q.QOQ_EPILOGUE_RESIDUAL)   # no residual
    with pytest.raises(q.QoQError):
        q.qoq_w4a8_gemm_fused(X8, s_x, packed, 7)
