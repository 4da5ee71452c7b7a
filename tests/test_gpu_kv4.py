"""KV4 decode attention with SmoothAttention, against the oracle, through the C ABI.

The cache writer (lambda, per-channel scales, packed codes) is bit-exact: it
rounds in the oracle's precision at every step.  The attention computes in
FP32 (the oracle in binary64); the bar is |err| <= 2 FP16 ulp of the oracle
value + 1e-3 of the output row's largest magnitude: FP32 sums over up to
2^20 tokens carry a relative error of a few 1e-7 per step, far inside one
FP16 ulp (2^-11), and the absolute term covers outputs that cancel to near
zero.  Shapes span grouped-query ratios 1-8, one token, ragged chunk tails
and long contexts split over many chunks.
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


def _codes(packed):
    """uint8 [.., L, d/2] nibbles -> int8 [.., L, d] codes."""
    p = packed.cpu().numpy()
    lo = (p & 0xF).astype(np.int8) - 8
    hi = (p >> 4).astype(np.int8) - 8
    return np.stack([lo, hi], axis=-1).reshape(*p.shape[:-1], p.shape[-1] * 2)


CASES = [(1, 4, 1, 1), (2, 8, 2, 37), (3, 32, 8, 1000), (1, 8, 8, 2048), (2, 16, 2, 4099), (1, 8, 4, 33000)]


@pytest.mark.parametrize("B,Hq,Hkv,L", CASES)
def test_kv4_cache_and_attention(B, Hq, Hkv, L):
    d = 128
    K, V = wl.make_kv(B, Hkv, L, d, seed=L + B)
    Q = wl.make_queries(B, Hq, d, seed=L + 7)
    cache = q.qoq_kv4_cache_quantize(K.cuda(), V.cuda())
    out = q.qoq_kv4_decode_attention(Q.cuda(), cache)
    torch.cuda.synchronize()
    got = _u16(out).view(np.float16).astype(np.float64)
    kc, vc = _codes(cache.K4), _codes(cache.V4)
    for b in range(B):
        r = oracle.kv4_decode(Q[b].numpy(), K[b].numpy(), V[b].numpy())
        assert np.array_equal(_u16(cache.lam)[b], r["lam"])
        assert np.array_equal(_u16(cache.s_k)[b], r["s_k"])
        assert np.array_equal(_u16(cache.s_v)[b], r["s_v"])
        assert np.array_equal(kc[b], r["k_codes"])
        assert np.array_equal(vc[b], r["v_codes"])
        ref = r["out"].view(np.float16).astype(np.float64)
        ulp = np.spacing(np.abs(ref).astype(np.float16)).astype(np.float64)
        tol = 2 * ulp + 1e-3 * np.abs(ref).max(axis=1, keepdims=True)
        bad = np.abs(got[b] - ref) > tol
        assert not bad.any(), f"sequence {b}: {bad.sum()} outputs beyond the bar"


def test_kv4_repeated_calls_identical_and_workspace_reuse():
    K, V = wl.make_kv(2, 4, 700, 128, seed=3)
    Q = wl.make_queries(2, 16, 128, seed=4)
    cache = q.qoq_kv4_cache_quantize(K.cuda(), V.cuda())
    ws = torch.full((q.qoq_kv4_attention_workspace_bytes(2, 16, 4, 700, 128),), 0x7f, dtype=torch.uint8,
                    device="cuda")
    o0 = q.qoq_kv4_decode_attention(Q.cuda(), cache, workspace=ws)
    for _ in range(3):
        assert torch.equal(q.qoq_kv4_decode_attention(Q.cuda(), cache, workspace=ws).view(torch.int16),
                           o0.view(torch.int16))


def test_kv4_rejects_bad_shapes():
    L = q.lib()
    A = torch.zeros(64, dtype=torch.uint8, device="cuda")
    p = A.data_ptr()
    import ctypes
    P = ctypes.c_void_p(p)
    assert q.qoq_kv4_attention_workspace_bytes(1, 12, 8, 16, 128) == 0   # Hq not a multiple of Hkv
    assert q.qoq_kv4_attention_workspace_bytes(1, 48, 3, 16, 128) == 0   # G = 16
    assert q.qoq_kv4_attention_workspace_bytes(1, 8, 8, 16, 64) == 0     # d != 128
    st = L.qoq_kv4_decode_attention(P, P, P, P, P, P, 1, 8, 8, 16, 128, P, P, 16, None)
    assert st == q.QOQ_ERR_INVALID_ARG                                    # workspace too small
