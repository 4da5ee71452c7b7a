"""Reference packing of canonical UINT4 codes into the documented packed
layout (include/qoq.h, "Packed weight layout"), written from that text with
numpy, independent of the CUDA packer."""
import numpy as np


def pack_reference(q: np.ndarray) -> np.ndarray:
    """q: uint8 [N][K] codes 0..15 -> uint8 [N*K/2] packed bytes."""
    N, K = q.shape
    assert N % 128 == 0 and K % 128 == 0
    # q[p*128 + r][b*128 + j*32 + h*16 + w*4 + i]  (h = 0: low nibble, 1: high)
    t = q.reshape(N // 128, 128, K // 128, 4, 2, 4, 4)      # p r b j h w i
    t = t.transpose(0, 2, 3, 1, 5, 6, 4)                    # p b j r w i h
    out = (t[..., 0] | (t[..., 1] << 4)).astype(np.uint8)   # p b j r w i
    return np.ascontiguousarray(out).reshape(-1)


def tables_reference(t: np.ndarray) -> np.ndarray:
    """Canonical group table [N][K/G] -> the documented panel-major layout
    [N/128][K/G][128] (include/qoq.h)."""
    N, ng = t.shape
    return np.ascontiguousarray(t.reshape(N // 128, 128, ng).transpose(0, 2, 1))
