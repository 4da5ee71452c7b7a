"""Reference packing of canonical UINT4 codes into the documented packed
layout (include/qoq.h, "Packed weight layout"), written from that text with
numpy, independent of the CUDA packer."""
import numpy as np


def pack_reference(q: np.ndarray, group_size: int, s_g: np.ndarray = None, zs: np.ndarray = None) -> np.ndarray:
    """q: uint8 [N][K] codes 0..15; s_g, zs: canonical [N][K/G] tables.

    Returns the packed bytes: per (panel, 128-wide K block) chunk the 8192
    code bytes, followed (group_size == 128 only) by the block's s_g and zs
    for the panel's 128 channels."""
    N, K = q.shape
    assert N % 128 == 0 and K % 128 == 0
    # q[p*128 + r][b*128 + j*32 + h*16 + w*4 + i]  (h = 0: low nibble, 1: high)
    t = q.reshape(N // 128, 128, K // 128, 4, 2, 4, 4)      # p r b j h w i
    t = t.transpose(0, 2, 3, 1, 5, 6, 4)                    # p b j r w i h
    codes = (t[..., 0] | (t[..., 1] << 4)).astype(np.uint8)  # p b j r w i
    codes = codes.reshape(N // 128, K // 128, 8192)
    if group_size != 128:
        return np.ascontiguousarray(codes).reshape(-1)
    assert s_g is not None and zs is not None and s_g.shape == (N, K // 128)
    sg = s_g.reshape(N // 128, 128, K // 128).transpose(0, 2, 1)   # p b r
    z = zs.reshape(N // 128, 128, K // 128).transpose(0, 2, 1)
    out = np.concatenate([codes, sg.astype(np.uint8), z.astype(np.uint8)], axis=2)
    return np.ascontiguousarray(out).reshape(-1)


def tables_reference(t: np.ndarray) -> np.ndarray:
    """Canonical group table [N][K/G] -> the documented panel-major layout
    [N/128][K/G][128] (include/qoq.h)."""
    N, ng = t.shape
    return np.ascontiguousarray(t.reshape(N // 128, 128, ng).transpose(0, 2, 1))
