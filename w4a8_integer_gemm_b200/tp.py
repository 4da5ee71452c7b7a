"""Row-parallel (K-split) W4A8 linear layer across GPUs.

Each of P ranks holds a contiguous slice [k0, k1) of the input dimension of
the packed weights (whole 128-wide K blocks, so every 128-wide group stays on
one rank).  The per-token activation quantization is computed from the whole
token row on every rank (X8 and s_x replicated, as the layer's input is), so
every rank's INT32 partial sums come from the same INT8 operands as the
single-GPU layer.  The partials are added with one all-reduce (an INT32 sum
is exact in any order) and the output scales are applied once after it:

    acc_r = X8[:, k0:k1] . W8hat[:, k0:k1]^T      (qoq_w4a8_gemm_i32, rank r)
    acc   = sum_r acc_r                           (all-reduce, INT32)
    Y     = fp16(((float)acc * s_x) * s_c)        (qoq_epilogue_i32)

The result is bit-identical to the single-GPU layer.  Sources: "QServe
Guide: W4A8KV4 Quantization for LLM Serving", The Architecture, subsection 2
(INT32 accumulation, scales applied once after the products); the pages list
multi-GPU tensor parallelism as open ("QServe: Low Bit Width Does Not
Guarantee High Throughput", section 12), so the partitioning is this
library's own.

This module only slices packed buffers (views and one strided copy at setup)
and calls the library's kernels and torch.distributed; it does no arithmetic
of the method itself.
"""
from __future__ import annotations

from typing import List, Optional, Tuple

import torch

from . import PackedWeights, qoq_epilogue_i32, qoq_w4a8_gemm_i32

BLOCK_K = 128          # K block of the packed layout (and the g128 group)
CHUNK_CODES = 8192     # code bytes of one (128-channel panel, K block) chunk
CHUNK_TABLES = 256     # s_g + zs of one chunk (g128 only)


def k_slices(K: int, world: int) -> List[Tuple[int, int]]:
    """[k0, k1) per rank: whole 128-wide K blocks, as even as they divide."""
    if K % BLOCK_K or world < 1:
        raise ValueError("K must be a multiple of 128 and world >= 1")
    blocks = K // BLOCK_K
    if blocks < world:
        raise ValueError(f"K = {K} has fewer 128-wide blocks than ranks ({world})")
    return [(BLOCK_K * (blocks * r // world), BLOCK_K * (blocks * (r + 1) // world)) for r in range(world)]


def shard_packed(packed: PackedWeights, k0: int, k1: int) -> PackedWeights:
    """The packed weights of input slice [k0, k1) (multiples of 128).

    With 128-wide groups each chunk carries its own tables, so the slice is
    chunks k0/128 .. k1/128 - 1 of every panel (one strided copy).  For the
    per-channel variant (one group per row) every slice keeps the row's
    tables and becomes its own one-group problem (group size = slice width,
    which must then be at least 256, since a 128-wide per-channel slice would
    read as the g128 layout)."""
    N, K, G = packed.N, packed.K, packed.group_size
    if k0 % BLOCK_K or k1 % BLOCK_K or not (0 <= k0 < k1 <= K):
        raise ValueError("the slice must be whole 128-wide K blocks inside [0, K)")
    per_group = G == BLOCK_K
    stride = CHUNK_CODES + (CHUNK_TABLES if per_group else 0)
    chunks = packed.Wp[: (N // 128) * (K // BLOCK_K) * stride].view(N // 128, K // BLOCK_K, stride)
    Wp = chunks[:, k0 // BLOCK_K: k1 // BLOCK_K, :].contiguous().view(-1)
    if per_group:
        s_g = packed.s_g[:, k0 // BLOCK_K: k1 // BLOCK_K, :].contiguous()
        zs = packed.zs[:, k0 // BLOCK_K: k1 // BLOCK_K, :].contiguous()
        G_local = BLOCK_K
    else:
        if k1 - k0 == BLOCK_K:
            raise ValueError("a per-channel slice must span at least 256 input channels")
        s_g, zs, G_local = packed.s_g, packed.zs, k1 - k0
    return PackedWeights(Wp, packed.s_c, s_g, zs, N, k1 - k0, G_local, packed.gate_up)


def allreduce_partials(acc: torch.Tensor, group=None) -> torch.Tensor:
    """Sum the ranks' INT32 partial sums in place (exact in any order)."""
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(acc, op=dist.ReduceOp.SUM, group=group)
    return acc


def linear_ksplit(X8: torch.Tensor, s_x: torch.Tensor, shard: PackedWeights, k0: int, s_c: torch.Tensor,
                  group=None, acc: Optional[torch.Tensor] = None, Y: Optional[torch.Tensor] = None,
                  workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """This rank's part of the row-parallel layer.

    X8: int8 [M, K_total] (every rank's copy), s_x its token scales; shard:
    this rank's slice from shard_packed starting at k0; s_c: the channel
    scales (the same on every rank).  Returns the full FP16 output [M, N]."""
    X8_local = X8[:, k0: k0 + shard.K]            # a view: the kernel takes the row stride
    acc = qoq_w4a8_gemm_i32(X8_local, shard, acc=acc, workspace=workspace, stream=stream)
    allreduce_partials(acc, group)
    return qoq_epilogue_i32(acc, s_x, s_c, Y=Y, stream=stream)
