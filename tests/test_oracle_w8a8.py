"""Pins of the W8A8 yardstick's weight quantizer (per-channel symmetric INT8,
FP16 scale max|W|/127, round half to even), against numpy and closed forms.

The pages name W8A8 as the INT8-peak yardstick of the roofline argument
("QServe: Low Bit Width Does Not Guarantee High Throughput", section 2,
Figure 3); they do not print its quantizer, so the plainest reading is used.
"""
import numpy as np

import oracle
from w4a8_integer_gemm_b200 import workloads as wl


def test_w8_matches_numpy_definition():
    W = wl.make_weights(64, 512, wl.LLAMA, seed=5).numpy()
    W8, s_w = oracle.quantize_weights_w8(W)
    amax = np.abs(W).max(axis=1).astype(np.float32)
    sw = (amax / np.float32(127.0)).astype(np.float32).astype(np.float16)
    assert np.array_equal(s_w, sw.view(np.uint16))
    q = np.rint(W / sw.astype(np.float32)[:, None]).clip(-127, 127).astype(np.int8)
    assert np.array_equal(W8, q)


def test_w8_properties_and_degenerate_rows():
    W = wl.make_weights(32, 256, wl.QWEN, seed=6).numpy()
    W[0] = 0.0
    W[1] = 1e-9                       # scale underflows to FP16 zero
    W8, s_w = oracle.quantize_weights_w8(W)
    assert np.all(W8[0] == 0) and s_w[0] == 0
    assert np.all(W8[1] == 0)
    top = np.abs(W8[2:].astype(int)).max(axis=1)
    assert np.all((top == 127) | (top == 126))          # the FP16 scale may round up
    sw = s_w[2:].view(np.float16).astype(np.float64)[:, None]
    err = np.abs(W8[2:] * sw - W[2:].astype(np.float64))
    assert np.all(err <= sw / 2 * (1 + 1e-6) + 1e-12)   # at most half a step


def test_w8a8_layer_against_fp64():
    X = wl.make_activations(5, 256, wl.LLAMA, seed=7)
    W = wl.make_weights(128, 256, wl.LLAMA, seed=8).numpy()
    r = oracle.linear_w8a8(X.numpy(), W)
    sx = r["s_x"].view(np.float16).astype(np.float64)
    sw = r["s_w"].view(np.float16).astype(np.float64)
    exact = (r["X8"].astype(np.float64) * sx[:, None]) @ (r["W8"].astype(np.float64) * sw[:, None]).T
    y = r["Y"].view(np.float16).astype(np.float64)
    ulp = np.spacing(np.abs(exact).astype(np.float16)).astype(np.float64)
    assert np.all(np.abs(y - exact) <= ulp)
