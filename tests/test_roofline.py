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


def test_mma_issue_ceiling():
    # 148 SMs x 8192 INT8 MACs per clock x 2 ops at 1965 MHz
    assert abs(roofline.mma_issue_ceiling_tops(1965.0) - 4764.8) < 0.1
    assert abs(roofline.mma_issue_ceiling_tops(1000.0, sms=1) - 16.384) < 1e-9


def test_regime_records_of_the_bench():
    """The bench's roofline record for each regime, from made-up timings
    (no GPU): the fields it reports and their arithmetic."""
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    if root not in sys.path:
        sys.path.insert(0, root)
    import bench
    from w4a8_integer_gemm_b200 import workloads as wl
    peaks = {"source": "measured", "hbm_gbs": 6543.4, "int8_tops": 3234.8, "int8_tops_sustained": 2745.4}
    sweep = wl.WORKLOADS["sweep"].shapes
    hbm = [s for s in sweep if s.M <= 128]
    ten = [s for s in sweep if s.M >= 256]
    traffic = {"sweep_M4096": {"dram_bytes": 352269824, "algorithmic_bytes": 135290880, "capture": "x",
                               "tensor_pipe_pct": 67.2}}
    r = bench.regime_roofline("tensor", ten, 0.9, peaks, traffic, 1965.0)
    ops = sum(roofline.ops(s.M, s.N, s.K) for s in ten)
    assert abs(r["achieved"] - ops / 0.9e-3 / 1e12) < 0.1
    assert abs(r["frac"] - r["achieved"] / 3234.8) < 1e-4
    assert abs(r["frac_of_mma_issue_ceiling"] - r["achieved"] / 4764.8) < 1e-4
    assert r["traffic"] == 352269824 and r["ncu_tensor_pipe_pct"] == 67.2 and r["launches"] == 6
    assert bench.regime_roofline("tensor", ten, 0.9, peaks, {}, None)["mma_issue_ceiling_tops"] == 4764.8
    h = bench.regime_roofline("hbm", hbm, 0.12, peaks, {}, 1965.0)
    byt = sum(roofline.algorithmic_bytes(s.M, s.N, s.K, s.G) for s in hbm)
    assert abs(h["achieved"] - byt / 0.12e-3 / 1e9) < 0.1 and "frac_of_mma_issue_ceiling" not in h
    assert "w4a8_gemv_kernel" in h["kernel"]
