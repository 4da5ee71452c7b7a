"""Pins of the oracle's stage 1, activation quantization, INT32 GEMM and
epilogue against properties, exact big-integer sums, FP64 matmuls and the
closed forms of the per-channel and g128 variants."""
import numpy as np
import pytest

import oracle
from w4a8_integer_gemm_b200 import workloads as wl


def _f16(bits):
    return np.asarray(bits, np.uint16).view(np.float16).astype(np.float64)


def test_stage1_properties():
    W = wl.make_weights(64, 1024, wl.LLAMA, seed=7).numpy()
    r = oracle.quantize_weights(W, 128)
    sc = _f16(r["s_c"])
    amax = np.abs(W).max(axis=1).astype(np.float64)
    # the scale is the FP16 value nearest to max|W|/119
    assert np.all(np.abs(sc - amax / 119) <= np.spacing(np.float16(amax / 119)).astype(np.float64) / 2 + 1e-12)
    # protective range: the largest magnitude lands on 119 exactly
    assert np.all(np.abs(r["W8"].astype(int)).max(axis=1) == 119)
    assert np.abs(r["W8"].astype(int)).max() <= 119
    # round to nearest: reconstruction error at most half a step
    err = np.abs(W.astype(np.float64) - sc[:, None] * r["W8"])
    assert np.all(err <= sc[:, None] * (0.5 + 1e-5))


def test_stage1_degenerate_rows():
    W = np.zeros((3, 256), np.float32)
    W[1, 5] = 1e-9           # scale underflows FP16 to zero -> row quantizes to zero
    W[2, :] = 1e-5           # subnormal FP16 scale (one 2^-24 step): values clamp to 119
    r = oracle.quantize_weights(W, 128)
    assert r["s_c"][0] == 0 and not r["W8"][0].any()
    assert r["s_c"][1] == 0 and not r["W8"][1].any()
    assert r["s_c"][2] == 1 and np.all(r["W8"][2] == 119)
    W8hat = oracle.dequant_weights(r["q"], r["s_g"], r["zs"], 128)
    assert not W8hat[0].any() and not W8hat[1].any()


def test_act_quant_properties():
    X = wl.make_activations(32, 4096, wl.LLAMA, seed=11).numpy()
    X8, s_x = oracle.quant_act(X)
    sx = _f16(s_x)
    assert np.all(np.abs(X8.astype(int)).max(axis=1) == 127)
    err = np.abs(X.astype(np.float64) - sx[:, None] * X8)
    assert np.all(err <= sx[:, None] * (0.5 + 1e-5))


def test_act_quant_degenerate_rows():
    X = np.zeros((3, 64), np.float16)
    X[1, :] = np.float16(6e-8)      # tiny row: FP16 scale rounds to zero
    X[2, 0] = np.float16(1e-4)      # subnormal scale: quotient may exceed 127 -> clamp
    X[2, 1] = np.float16(-1e-4)
    X8, s_x = oracle.quant_act(X)
    assert s_x[0] == 0 and not X8[0].any()
    assert s_x[1] == 0 and not X8[1].any()
    assert X8[2].max() <= 127 and X8[2].min() >= -128 and X8[2, 0] > 0 > X8[2, 1]


def test_gemm_exact_against_big_integers():
    rng = np.random.default_rng(3)
    X8 = rng.integers(-128, 128, size=(3, 384), dtype=np.int64).astype(np.int8)
    W8 = rng.integers(-127, 128, size=(5, 384), dtype=np.int64).astype(np.int8)
    acc = oracle.gemm_i32(X8, W8)
    for m in range(3):
        for n in range(5):
            assert int(acc[m, n]) == sum(int(a) * int(b) for a, b in zip(X8[m], W8[n]))


def test_int32_bound_at_largest_k():
    K = 24576
    X = np.ones((1, K), np.float16)
    W = np.stack([np.ones(K, np.float32), -np.ones(K, np.float32)])
    r = oracle.linear(X, W, 128)
    # W8 = +-119; group range 119 -> s_g = 8; codes give +-120
    assert set(np.unique(r["W8hat"])) == {-120, 120}
    assert list(r["acc"][0]) == [K * 127 * 120, -K * 127 * 120]
    assert np.abs(r["acc"].astype(np.int64)).max() <= K * 128 * 127 < 2**31


@pytest.mark.parametrize("G", [128, 512])
def test_output_against_fp64_dequantized_matmul(G):
    X = wl.make_activations(16, 512, wl.TINY, seed=5).numpy()
    W = wl.make_weights(512, 512, wl.TINY, seed=6).numpy()
    r = oracle.linear(X, W, G)
    sx, sc = _f16(r["s_x"]), _f16(r["s_c"])
    ref = (sx[:, None] * r["X8"].astype(np.float64)) @ (sc[:, None] * r["W8hat"].astype(np.float64)).T
    y = _f16(r["Y"])
    ulp = np.spacing(np.abs(ref).astype(np.float16)).astype(np.float64)
    assert np.all(np.abs(y - ref) <= ulp)
    # quality sanity (not parity): near the unquantized FP32 product.  The
    # synthetic weights carry x20 outlier input channels with no smoothing or
    # rotation (those need calibration data), so the bar is loose: about
    # 0.977 (g128) and 0.944 (per-channel) are what this distribution gives.
    full = X.astype(np.float64) @ W.astype(np.float64).T
    cos = (y * full).sum() / np.linalg.norm(y) / np.linalg.norm(full)
    assert cos > (0.95 if G == 128 else 0.90)


def _closed_form(X8, q, z, s_g, G):
    """acc = sum_g s_g * (X8_g . q_g - z_g * rowsum(X8_g))."""
    M, K = X8.shape
    acc = np.zeros((M, q.shape[0]), np.int64)
    x = X8.astype(np.int64)
    for g in range(K // G):
        sl = slice(g * G, (g + 1) * G)
        rs = x[:, sl].sum(axis=1)
        acc += (x[:, sl] @ q[:, sl].astype(np.int64).T - rs[:, None] * z[:, g].astype(np.int64)[None, :]) \
            * s_g[:, g].astype(np.int64)[None, :]
    return acc


@pytest.mark.parametrize("G", [128, 1024])
def test_closed_forms(G):
    X = wl.make_activations(8, 1024, wl.LLAMA, seed=21).numpy()
    W = wl.make_weights(96, 1024, wl.LLAMA, seed=22).numpy()
    r = oracle.linear(X, W, G)
    assert np.array_equal(r["acc"].astype(np.int64), _closed_form(r["X8"], r["q"], r["z"], r["s_g"], G))


def test_per_channel_equals_g128_when_groups_share_range():
    rng = np.random.default_rng(9)
    K = 1024
    W = (rng.standard_normal((16, K)) * 0.02).astype(np.float32)
    hi = np.abs(W).max(axis=1) * 1.5
    for g in range(K // 128):           # every group holds the row's max and min
        W[:, g * 128] = hi
        W[:, g * 128 + 1] = -hi * 0.9   # below every other entry (those are < hi/1.5)
    X = wl.make_activations(4, K, wl.LLAMA, seed=23).numpy()
    a = oracle.linear(X, W, K)
    b = oracle.linear(X, W, 128)
    assert np.array_equal(np.repeat(a["s_g"], K // 128, axis=1), b["s_g"])
    assert np.array_equal(a["q"], b["q"])
    assert np.array_equal(a["acc"], b["acc"])
    assert np.array_equal(a["Y"], b["Y"])


def test_group_must_divide_k():
    with pytest.raises(ValueError):
        oracle.quantize_weights(np.zeros((2, 100), np.float32), 128)
