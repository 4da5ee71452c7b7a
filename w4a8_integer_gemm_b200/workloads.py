"""Seeded synthetic inputs for the W4A8 linear layer, and the workload table.

This module holds no arithmetic of the method: it draws the FP32 master
weights W [N][K] and the FP16 activations X [M][K] that both the CUDA path and
the CPU oracle consume.  Shapes are the linear layers of Llama-3-8B and
Qwen1.5-72B (no model weights are used or needed: values are normal draws with
a fraction of input channels scaled up to make outliers).

Recipe (one torch CPU generator per tensor, so every draw is reproducible on
any machine):
  W = std * randn(N, K); then round(w_frac*K) input channels (columns k),
      picked by randperm without replacement, are multiplied by w_scale.
  X = randn(M, K) in FP32; then round(x_frac*K) columns are multiplied by
      x_scale; then cast to FP16 (round to nearest even).
  Seeds: workload number c, shape index i -> W seed 1000*c + 2*i,
         X seed 1000*c + 2*i + 1.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import List, Tuple

import torch


@dataclass(frozen=True)
class Dist:
    w_std: float
    w_frac: float
    w_scale: float
    x_frac: float
    x_scale: float


# Weight / activation distributions named by the workloads.
TINY = Dist(w_std=0.02, w_frac=0.02, w_scale=20.0, x_frac=0.0, x_scale=1.0)
LLAMA = Dist(w_std=0.02, w_frac=0.01, w_scale=20.0, x_frac=0.005, x_scale=50.0)
QWEN = Dist(w_std=0.015, w_frac=0.01, w_scale=25.0, x_frac=0.005, x_scale=50.0)


@dataclass(frozen=True)
class Shape:
    M: int
    K: int
    N: int
    G: int          # group size: 128, or K for the per-channel variant
    name: str


@dataclass
class Workload:
    number: int
    name: str
    dist: Dist
    shapes: List[Shape] = field(default_factory=list)

    def seeds(self, i: int) -> Tuple[int, int]:
        return 1000 * self.number + 2 * i, 1000 * self.number + 2 * i + 1


def _workloads() -> dict:
    w = {}
    w["tiny"] = Workload(1, "tiny_16x512x512_g128", TINY,
                         [Shape(16, 512, 512, 128, "tiny")])
    dec = []
    for G in (4096, 128):
        for M in (1, 8, 32, 64):
            tag = "pc" if G == 4096 else "g128"
            dec.append(Shape(M, 4096, 14336, G, f"llama3_8b_up_M{M}_{tag}"))
    w["decode"] = Workload(2, "decode_llama3_8b_up_K4096_N14336", LLAMA, dec)
    lb = []
    for M in (256, 1024, 4096):
        for (K, N, nm) in ((4096, 6144, "qkv"), (4096, 4096, "o"),
                           (4096, 28672, "gate_up"), (14336, 4096, "down")):
            lb.append(Shape(M, K, N, 128, f"llama3_8b_{nm}_M{M}"))
    w["large_batch"] = Workload(3, "large_batch_llama3_8b_linears", LLAMA, lb)
    qw = []
    for M in (64, 512, 2048):
        for (K, N, nm) in ((8192, 24576, "up"), (24576, 8192, "down"), (8192, 8192, "o")):
            for G in (K, 128):
                tag = "pc" if G == K else "g128"
                qw.append(Shape(M, K, N, G, f"qwen15_72b_{nm}_M{M}_{tag}"))
    w["qwen"] = Workload(4, "qwen15_72b_linears", QWEN, qw)
    sw = [Shape(1 << e, 8192, 8192, 128, f"sweep_M{1 << e}") for e in range(14)]
    w["sweep"] = Workload(5, "batch_sweep_K8192_N8192_g128", LLAMA, sw)
    return w


WORKLOADS = _workloads()


def _outlier_columns(K: int, frac: float, gen: torch.Generator) -> torch.Tensor:
    count = int(round(frac * K))
    return torch.randperm(K, generator=gen)[:count]


def make_weights(N: int, K: int, dist: Dist, seed: int) -> torch.Tensor:
    """FP32 master weights [N][K] on the CPU."""
    gen = torch.Generator(device="cpu").manual_seed(int(seed))
    W = torch.randn(N, K, generator=gen, dtype=torch.float32) * dist.w_std
    cols = _outlier_columns(K, dist.w_frac, gen)
    if cols.numel():
        W[:, cols] *= dist.w_scale
    return W


def make_activations(M: int, K: int, dist: Dist, seed: int) -> torch.Tensor:
    """FP16 activations [M][K] on the CPU."""
    gen = torch.Generator(device="cpu").manual_seed(int(seed))
    X = torch.randn(M, K, generator=gen, dtype=torch.float32)
    cols = _outlier_columns(K, dist.x_frac, gen)
    if cols.numel():
        X[:, cols] *= dist.x_scale
    return X.to(torch.float16)


def make_kv(B: int, Hkv: int, L: int, d: int, seed: int, k_frac: float = 0.02, k_scale: float = 25.0):
    """FP16 keys and values [B, Hkv, L, d] of a synthetic KV cache: normal
    draws, with round(k_frac * d) key channels per KV head (picked without
    replacement) scaled by k_scale, the outlier channels SmoothAttention is
    for."""
    gen = torch.Generator(device="cpu").manual_seed(int(seed))
    K = torch.randn(B, Hkv, L, d, generator=gen, dtype=torch.float32)
    V = torch.randn(B, Hkv, L, d, generator=gen, dtype=torch.float32)
    count = int(round(k_frac * d))
    for h in range(Hkv):
        cols = torch.randperm(d, generator=gen)[:count]
        if count:
            K[:, h, :, cols] *= k_scale
    return K.to(torch.float16), V.to(torch.float16)


def make_queries(B: int, Hq: int, d: int, seed: int):
    """FP16 queries [B, Hq, d] (one new token per sequence)."""
    gen = torch.Generator(device="cpu").manual_seed(int(seed))
    return torch.randn(B, Hq, d, generator=gen, dtype=torch.float32).to(torch.float16)


def make_case(workload: Workload, i: int, shape: Shape = None):
    """(X fp16 [M][K], W fp32 [N][K]) for shape i of a workload."""
    s = shape or workload.shapes[i]
    sw, sx = workload.seeds(i)
    return make_activations(s.M, s.K, workload.dist, sx), make_weights(s.N, s.K, workload.dist, sw)
