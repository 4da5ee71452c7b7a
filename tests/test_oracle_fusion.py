"""Pins of the oracle's output-side fusions against independent definitions.

The residual add and the SiLU-gated product follow the layer (the pages
describe the layer's epilogue, "QServe Guide: W4A8KV4 Quantization for LLM
Serving", The Architecture, subsection 2, but not the ops after it).  The
reading taken is that a fused epilogue returns exactly what the unfused ops
return.  These tests check the oracle's C code against numpy's own IEEE
conversions and arithmetic, and against closed-form special cases.
"""
import numpy as np
import pytest

import oracle


def _rng(seed):
    return np.random.default_rng(seed)


def test_double_to_half_matches_numpy():
    r = _rng(1)
    x = np.concatenate([
        r.standard_normal(40000) * 10.0 ** r.integers(-9, 5, 40000),
        # exact midpoints between adjacent halves (ties) and their neighbours
        (np.arange(0, 65504, dtype=np.float16)[::97].astype(np.float64)
         + np.spacing(np.arange(0, 65504, dtype=np.float16)[::97]).astype(np.float64) / 2),
        np.array([0.0, -0.0, 65504.0, 65519.99, 65520.0, 1e9, -1e9, 2.0 ** -24, 2.0 ** -25,
                  3 * 2.0 ** -26, 2.0 ** -14, 2.0 ** -14 - 2.0 ** -25]),
    ])
    x = np.concatenate([x, -x])
    want = x.astype(np.float16).view(np.uint16)
    got = np.array([oracle.double_to_half_bits(v) for v in x], dtype=np.uint16)
    assert np.array_equal(got, want)


def _layer_inputs(seed, M, N, amax=2 ** 24):
    r = _rng(seed)
    acc = r.integers(-amax, amax, size=(M, N), dtype=np.int64).astype(np.int32)
    s_x = (r.random(M) * 0.05 + 1e-4).astype(np.float16).view(np.uint16)
    s_c = (r.random(N) * 1e-3 + 1e-6).astype(np.float16).view(np.uint16)
    return acc, s_x, s_c


def _layer_y_numpy(acc, s_x, s_c):
    """The layer's FP16 output with numpy float32 arithmetic (no FMA)."""
    sx = s_x.view(np.float16).astype(np.float32)[:, None]
    sc = s_c.view(np.float16).astype(np.float32)[None, :]
    return ((acc.astype(np.float32) * sx) * sc).astype(np.float16)


def test_residual_matches_numpy_fp16_add():
    acc, s_x, s_c = _layer_inputs(2, 37, 96)
    R = (_rng(3).standard_normal((37, 96)) * 4).astype(np.float16)
    got = oracle.epilogue_residual(acc, s_x, s_c, R)
    y = _layer_y_numpy(acc, s_x, s_c)
    want = (y.astype(np.float32) + R.astype(np.float32)).astype(np.float16).view(np.uint16)
    assert np.array_equal(got, want)
    # the layer's own epilogue is the plain-epilogue special case
    assert np.array_equal(oracle.epilogue(acc, s_x, s_c), y.view(np.uint16))


def test_residual_special_cases():
    acc, s_x, s_c = _layer_inputs(4, 8, 32)
    plain = oracle.epilogue(acc, s_x, s_c)
    zero = np.zeros((8, 32), np.float16)
    assert np.array_equal(oracle.epilogue_residual(acc, s_x, s_c, zero), plain)
    # adding the negated output gives exact zeros
    neg = (-plain.view(np.float16))
    out = oracle.epilogue_residual(acc, s_x, s_c, neg).view(np.float16)
    assert np.all(out == 0)


def test_silu_mul_matches_numpy_float64():
    acc, s_x, s_c = _layer_inputs(5, 19, 256, amax=2 ** 20)
    got = oracle.epilogue_silu_mul(acc, s_x, s_c)
    y = _layer_y_numpy(acc, s_x, s_c).astype(np.float64)
    g, u = y[:, :128], y[:, 128:]
    want = (g / (1.0 + np.exp(-g)) * u).astype(np.float16).view(np.uint16)
    assert np.array_equal(got, want)


def test_silu_mul_pairs_gate_j_with_up_j():
    """Only column j of the gate half and column I + j of the up half meet:
    a swapped or shifted pairing fails here."""
    M, I = 3, 64
    acc = np.zeros((M, 2 * I), np.int32)
    s_x = np.full(M, np.float16(1.0)).view(np.uint16)
    s_c = np.full(2 * I, np.float16(1.0)).view(np.uint16)
    j = np.arange(I)
    acc[:, j] = 20 + j           # gate: large, so silu(g) = g exactly in FP16 terms
    acc[:, I + j] = 2 + (j % 7)  # up
    out = oracle.epilogue_silu_mul(acc, s_x, s_c).view(np.float16).astype(np.float64)
    g = (20 + j).astype(np.float64)
    want = (g / (1 + np.exp(-g)) * (2 + (j % 7))).astype(np.float16).astype(np.float64)
    assert np.array_equal(out, np.broadcast_to(want, (M, I)))


@pytest.mark.parametrize("gval,uval,expect", [(0.0, 3.0, 0.0), (2.5, 0.0, 0.0), (-30.0, 2.0, 0.0)])
def test_silu_mul_closed_forms(gval, uval, expect):
    s_x = np.full(1, np.float16(1.0)).view(np.uint16)
    s_c = np.full(2, np.float16(0.5)).view(np.uint16)
    acc = np.array([[int(gval * 2), int(uval * 2)]], np.int32)
    out = oracle.epilogue_silu_mul(acc, s_x, s_c).view(np.float16).astype(np.float64)
    assert abs(out[0, 0] - expect) < 1e-10
