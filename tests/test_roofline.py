"""Pins the roofline time model to the crossover the pages print for A100."""
import os

from w4a8_integer_gemm_b200 import roofline

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "a100_roofline_crossover.txt")


def test_a100_crossover_matches_pages():
    d = {}
    for line in open(GOLDEN):
        line = line.strip()
        if line and not line.startswith("#"):
            k, v = line.split(":")
            d[k.strip()] = float(v)
    bw = d["dram_tbs"] * 1e12
    w4a16 = (d["fp16_tops"] * 1e12, d["w4a16_bytes_per_weight"])
    w8a8 = (d["int8_tops"] * 1e12, d["w8a8_bytes_per_weight"])
    assert roofline.crossover_m(w4a16, w8a8, bw) == int(d["crossover_m"])


def test_bytes_and_bound():
    # decode: weights dominate; K=4096, N=14336, g128 -> 29.36 MB + tables
    b = roofline.algorithmic_bytes(1, 14336, 4096, 128)
    assert b == 14336 * 2048 + 2 * 14336 * 32 + 2 * 14336 + 4096 + 2 + 2 * 14336
    assert roofline.bound(1, 14336, 4096, 128, 3.2e15, 6.5e12) == "hbm"
    assert roofline.bound(4096, 8192, 8192, 128, 3.2e15, 6.5e12) == "tensor"
    assert roofline.ops(2, 3, 5) == 60
