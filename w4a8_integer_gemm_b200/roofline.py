"""Roofline model of the W4A8 GEMM (measurement code, not the method).

Algorithmic bytes of one GEMM: the packed 4-bit weights, the two 8-bit group
tables (integer scale s_g and zero compensation z*s_g), the FP16 channel
scales, the INT8 activations with their FP16 token scales, and the FP16
output:

    bytes = N*K/2 + 2*N*(K/G) + 2*N + M*K + 2*M + 2*M*N
    ops   = 2*M*N*K

The roofline is min(INT8 dense peak, ops * HBM bandwidth / bytes): the GEMM is
bandwidth-bound for small M (decode) and tensor-bound for large M.  The same
time model t(m) = max(ops/peak, bytes/bandwidth), restricted to weight bytes,
reproduces the A100 crossover the pages quote ("QServe: Low Bit Width Does Not
Guarantee High Throughput", section 2 "Motivation": W4A16 favourable below
m of about 78 on A100 with 312/624 TOPS FP16/INT8 and about 2 TB/s).
"""
from __future__ import annotations

import json
import os


def algorithmic_bytes(M: int, N: int, K: int, G: int) -> int:
    return N * K // 2 + 2 * N * (K // G) + 2 * N + M * K + 2 * M + 2 * M * N


def algorithmic_bytes_w8(M: int, N: int, K: int) -> int:
    """The W8A8 yardstick: INT8 weights and their FP16 channel scales, X8 with
    its token scales, FP16 Y."""
    return N * K + 2 * N + M * K + 2 * M + 2 * M * N


def act_quant_bytes(M: int, K: int) -> int:
    """FP16 X read, INT8 X8 written, FP16 s_x written."""
    return 2 * M * K + M * K + 2 * M


def ops(M: int, N: int, K: int) -> int:
    return 2 * M * N * K


def roofline_ops_per_s(M: int, N: int, K: int, G: int, peak_ops: float, bw_bytes: float) -> float:
    return min(peak_ops, ops(M, N, K) * bw_bytes / algorithmic_bytes(M, N, K, G))


def bound(M: int, N: int, K: int, G: int, peak_ops: float, bw_bytes: float) -> str:
    t_c = ops(M, N, K) / peak_ops
    t_m = algorithmic_bytes(M, N, K, G) / bw_bytes
    return "tensor" if t_c >= t_m else "hbm"


def weight_stream_time(m: float, peak_ops: float, bytes_per_weight: float, bw_bytes: float) -> float:
    """Time per weight element of an m-token GEMM when only weights move."""
    return max(2.0 * m / peak_ops, bytes_per_weight / bw_bytes)


def crossover_m(fmt_a, fmt_b, bw_bytes: float, m_max: int = 1 << 16) -> int:
    """Smallest integer m at which format a is no faster than format b.

    fmt = (peak ops/s, bytes per weight element)."""
    for m in range(1, m_max):
        ta = weight_stream_time(m, fmt_a[0], fmt_a[1], bw_bytes)
        tb = weight_stream_time(m, fmt_b[0], fmt_b[1], bw_bytes)
        if ta >= tb:
            return m
    return m_max


# The INT8 MMA issue rate measured on this part: one tcgen05.mma kind::i8
# of 128 x 256 x 32 per 128 SM cycles (one thread issuing back to back),
# i.e. 8192 multiply-adds per clock per SM.  A second ceiling for the
# tensor-bound GEMM beside the BF16-derived peak: it scales with the SM
# clock the kernel actually ran at.
MMA_I8_MACS_PER_CLK_PER_SM = 8192
SMS = 148


def mma_issue_ceiling_tops(sm_mhz: float, sms: int = SMS) -> float:
    """INT8 ops/s (in TOPS) at the measured MMA issue rate and this SM clock."""
    return sms * MMA_I8_MACS_PER_CLK_PER_SM * 2 * sm_mhz * 1e6 / 1e12


# ---------------------------------------------------------------- peaks ----
# Nominal dense ratio INT8 : BF16 on B200 (4.5 : 2.25 PFLOP/s).
INT8_PER_BF16 = 2.0
FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks(path: str = None) -> dict:
    """Measured HBM GB/s and dense INT8 TOPS (burst and sustained).

    INT8 peaks are the measured BF16 GEMM peaks times the nominal INT8:BF16
    ratio of 2; 'source' says whether the measured file or the fallback
    figures were used."""
    if path is None:
        path = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                            "MEASURED_PEAKS.json")
    src = "measured"
    try:
        with open(path) as f:
            p = json.load(f)
    except (OSError, ValueError):
        p, src = dict(FALLBACK), "fallback"
    bf16 = float(p.get("bf16_tflops", FALLBACK["bf16_tflops"]))
    bf16s = float(p.get("bf16_tflops_sustained", FALLBACK["bf16_tflops_sustained"]))
    return {
        "source": src,
        "hbm_gbs": float(p.get("hbm_gbs", FALLBACK["hbm_gbs"])),
        "int8_tops": bf16 * INT8_PER_BF16,
        "int8_tops_sustained": bf16s * INT8_PER_BF16,
    }
