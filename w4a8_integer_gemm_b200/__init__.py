"""B200-native QoQ W4A8 linear layer: Y = diag(s_x) (X8 W8hat^T) diag(s_c).

A thin ctypes binding over libqoq.so (include/qoq.h).  Every function here
has the name of the C entry point it calls and only marshals arguments:
torch tensors provide device memory and the current CUDA stream, every step
of the computation runs in the library's sm_100a kernels.  There is no CPU
fallback: if the shared library is missing or the device is not a B200, the
calls raise.

    packed = qoq_pack_weights(W_fp32_cuda, group_size)        # offline
    X8, s_x = qoq_quant_act_per_token(X_fp16_cuda)            # per forward
    Y = qoq_w4a8_gemm(X8, s_x, packed)                        # per forward

`W4A8Linear` wraps the three for a layer; `w4a8_linear_host` is the end to
end call a user makes with host tensors, and `w4a8_linear_host_many` runs
several of them with their host copies overlapping the kernels.
"""
from __future__ import annotations

import ctypes
import os
import threading
from dataclasses import dataclass
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libqoq.so")

QOQ_OK = 0
QOQ_ERR_INVALID_ARG = -1
QOQ_ERR_UNSUPPORTED = -2
QOQ_ERR_CUDA = -3
QOQ_ERR_TIMEOUT = -4
QOQ_ERR_SCRATCH_TOO_SMALL = -5
QOQ_NOALLOC_SCRATCH_BYTES = 16 << 20
QOQ_EPILOGUE_NONE = 0
QOQ_EPILOGUE_RESIDUAL = 1
QOQ_EPILOGUE_SILU_MUL = 2

_P = ctypes.c_void_p
_I = ctypes.c_int
_SZ = ctypes.c_size_t

# name -> (restype, argtypes); the exported surface of include/qoq.h
SIGNATURES = {
    "qoq_status_string": (ctypes.c_char_p, [_I]),
    "qoq_packed_weight_bytes": (_SZ, [_I, _I, _I]),
    "qoq_pack_weights": (_I, [_P, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P]),
    "qoq_pack_weights_gate_up": (_I, [_P, _I, _I, _I, _P, _P, _P, _P, _P]),
    "qoq_quant_act_per_token": (_I, [_P, _I, _I, _P, _P, _P, _P]),
    "qoq_gemm_workspace_bytes": (_SZ, [_I, _I, _I, _I]),
    "qoq_w4a8_gemm": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _P, _P, _P, _SZ, _P]),
    "qoq_w4a8_gemm_noalloc": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _P, _P]),
    "qoq_w4a8_gemm_fused": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _P, _P, _P, _SZ, _P]),
    "qoq_w4a8_gemm_i32": (_I, [_P, _I, _P, _P, _P, _I, _I, _I, _I, _P, _P, _SZ, _P]),
    "qoq_epilogue_i32": (_I, [_P, _P, _P, _I, _I, _P, _P]),
    "qoq_quantize_weights_w8": (_I, [_P, _I, _I, _P, _P, _P]),
    "qoq_kv4_cache_quantize": (_I, [_P, _P, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P]),
    "qoq_kv4_attention_workspace_bytes": (_SZ, [_I, _I, _I, _I, _I]),
    "qoq_kv4_decode_attention": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _P, _P, _SZ, _P]),
    "qoq_w8a8_gemm": (_I, [_P, _P, _P, _P, _I, _I, _I, _P, _P, _P, _SZ, _P]),
    "qoq_w4a8_linear": (_I, [_P, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P, _P, _SZ, _P]),
    "qoq_dequant_weights_i8": (_I, [_P, _P, _P, _I, _I, _I, _P, _P]),
    "qoq_set_gemm_a_in_tmem": (_I, [_I]),
    "qoq_set_gemm_cta_pairs": (_I, [_I]),
    "qoq_set_gemm_narrow_tiles": (_I, [_I]),
    "qoq_set_gemm_half_ctas": (_I, [_I]),
    "qoq_set_gemm_gemv": (_I, [_I]),
    "qoq_set_linear_in_kernel_quant": (_I, [_I]),
    "qoq_selftest_wait_timeout": (_I, [ctypes.c_ulonglong, _P]),
    "qoq_device_error": (_I, [_P]),
}

_lock = threading.Lock()
_lib = None


class QoQError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn} failed: {status} ({qoq_status_string(status)})")


def lib() -> ctypes.CDLL:
    """The loaded libqoq.so.  Raises if it has not been built."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(
                    f"libqoq.so not found at {LIB_PATH}; build it with "
                    "`python -m w4a8_integer_gemm_b200.build_lib` (there is no CPU fallback)")
            L = ctypes.CDLL(LIB_PATH)
            for name, (res, args) in SIGNATURES.items():
                f = getattr(L, name)
                f.restype = res
                f.argtypes = args
            _lib = L
        return _lib


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def _check(fn: str, status: int):
    if status != QOQ_OK:
        raise QoQError(fn, status)


def _need(t: torch.Tensor, dtype, name):
    if not (t.is_cuda and t.dtype == dtype and t.is_contiguous()):
        raise ValueError(f"{name} must be a contiguous CUDA {dtype} tensor")


# ------------------------------------------------------------------ ABI ----
def qoq_status_string(status: int) -> str:
    return lib().qoq_status_string(int(status)).decode()


def qoq_packed_weight_bytes(N: int, K: int, group_size: int) -> int:
    return int(lib().qoq_packed_weight_bytes(int(N), int(K), int(group_size)))


def qoq_gemm_workspace_bytes(M: int, N: int, K: int, group_size: int) -> int:
    return int(lib().qoq_gemm_workspace_bytes(int(M), int(N), int(K), int(group_size)))


def qoq_set_gemm_a_in_tmem(enable: bool) -> None:
    _check("qoq_set_gemm_a_in_tmem", lib().qoq_set_gemm_a_in_tmem(1 if enable else 0))


def qoq_set_gemm_cta_pairs(enable: bool) -> None:
    _check("qoq_set_gemm_cta_pairs", lib().qoq_set_gemm_cta_pairs(1 if enable else 0))


def qoq_set_gemm_narrow_tiles(enable: bool) -> None:
    _check("qoq_set_gemm_narrow_tiles", lib().qoq_set_gemm_narrow_tiles(1 if enable else 0))


def qoq_set_gemm_half_ctas(enable: bool) -> None:
    _check("qoq_set_gemm_half_ctas", lib().qoq_set_gemm_half_ctas(1 if enable else 0))


def qoq_set_gemm_gemv(enable: bool) -> None:
    """M <= 8 tokens: the decode kernel (warp-level INT8 MMAs; True, the default) or the tensor-core GEMM."""
    _check("qoq_set_gemm_gemv", lib().qoq_set_gemm_gemv(1 if enable else 0))


def qoq_set_linear_in_kernel_quant(enable: bool) -> None:
    _check("qoq_set_linear_in_kernel_quant", lib().qoq_set_linear_in_kernel_quant(1 if enable else 0))


def qoq_selftest_wait_timeout(timeout_ns: int, stream=None) -> None:
    """Launch one bounded wait that nothing completes (the failure-path self-test)."""
    _check("qoq_selftest_wait_timeout", lib().qoq_selftest_wait_timeout(int(timeout_ns), _stream(stream)))


def qoq_device_error(stream=None) -> int:
    """QOQ_OK, or QOQ_ERR_TIMEOUT if a GEMM's bounded wait ran out."""
    return int(lib().qoq_device_error(_stream(stream)))


@dataclass
class PackedWeights:
    """Output of the offline packer (device tensors, layouts of include/qoq.h)."""
    Wp: torch.Tensor     # uint8 [N*K/2]  interleaved UINT4 codes
    s_c: torch.Tensor    # int16 [N]      FP16 bits of the channel scales
    s_g: torch.Tensor    # uint8 [N/128, K/G, 128] integer group scales (panel-major)
    zs: torch.Tensor     # uint8 [N/128, K/G, 128] zero compensation z*s_g
    N: int
    K: int
    group_size: int
    gate_up: bool = False   # packed by qoq_pack_weights_gate_up (64 gate + 64 up channels per panel)


def qoq_pack_weights(W: torch.Tensor, group_size: int, out: Optional[PackedWeights] = None,
                     stream=None, z_dbg: Optional[torch.Tensor] = None,
                     q_dbg: Optional[torch.Tensor] = None) -> PackedWeights:
    """W fp32 [N, K] -> packed weights.  z_dbg (uint8 [N, K/G]) and q_dbg
    (uint8 [N, K]), when given, receive the zero points and the canonical
    codes for inspection."""
    _need(W, torch.float32, "W")
    if z_dbg is not None:
        _need(z_dbg, torch.uint8, "z_dbg")
    if q_dbg is not None:
        _need(q_dbg, torch.uint8, "q_dbg")
    N, K = W.shape
    G = int(group_size)
    if out is None:
        dev = W.device
        nb = qoq_packed_weight_bytes(N, K, G)
        ng = K // G if G > 0 and K % G == 0 else 1
        out = PackedWeights(torch.empty(max(nb, 16), dtype=torch.uint8, device=dev),
                            torch.empty(N, dtype=torch.int16, device=dev),
                            torch.empty(max(N // 128, 1), ng, 128, dtype=torch.uint8, device=dev),
                            torch.empty(max(N // 128, 1), ng, 128, dtype=torch.uint8, device=dev), N, K, G)
    st = lib().qoq_pack_weights(_ptr(W), N, K, G, _ptr(out.Wp), _ptr(out.s_c), _ptr(out.s_g),
                                _ptr(out.zs), _ptr(z_dbg), _ptr(q_dbg), _stream(stream))
    _check("qoq_pack_weights", st)
    return out


def qoq_pack_weights_gate_up(W: torch.Tensor, group_size: int, stream=None) -> PackedWeights:
    """W fp32 [N, K] = [gate rows; up rows] -> packed weights whose panels
    hold 64 gate channels and the 64 matching up channels, for the SiLU-gated
    epilogue of qoq_w4a8_gemm_fused."""
    _need(W, torch.float32, "W")
    N, K = W.shape
    G = int(group_size)
    dev = W.device
    nb = qoq_packed_weight_bytes(N, K, G)
    ng = K // G if G > 0 and K % G == 0 else 1
    out = PackedWeights(torch.empty(max(nb, 16), dtype=torch.uint8, device=dev),
                        torch.empty(N, dtype=torch.int16, device=dev),
                        torch.empty(max(N // 128, 1), ng, 128, dtype=torch.uint8, device=dev),
                        torch.empty(max(N // 128, 1), ng, 128, dtype=torch.uint8, device=dev), N, K, G, True)
    st = lib().qoq_pack_weights_gate_up(_ptr(W), N, K, G, _ptr(out.Wp), _ptr(out.s_c), _ptr(out.s_g),
                                        _ptr(out.zs), _stream(stream))
    _check("qoq_pack_weights_gate_up", st)
    return out


def qoq_quant_act_per_token(X: torch.Tensor, X8: Optional[torch.Tensor] = None,
                            s_x: Optional[torch.Tensor] = None, stream=None,
                            rowsum: Optional[torch.Tensor] = None):
    """X fp16 [M, K] -> (X8 int8 [M, K], s_x int16 [M] FP16 bits).  rowsum
    (int32 [M]), when given, receives sum_k X8[m, k]."""
    _need(X, torch.float16, "X")
    if rowsum is not None:
        _need(rowsum, torch.int32, "rowsum")
    M, K = X.shape
    if X8 is None:
        X8 = torch.empty(M, K, dtype=torch.int8, device=X.device)
    if s_x is None:
        s_x = torch.empty(max(M, 8), dtype=torch.int16, device=X.device)
    st = lib().qoq_quant_act_per_token(_ptr(X), M, K, _ptr(X8), _ptr(s_x), _ptr(rowsum), _stream(stream))
    _check("qoq_quant_act_per_token", st)
    return X8, s_x


_ws_cache = {}


def gemm_workspace(M: int, N: int, K: int, group_size: int, device) -> torch.Tensor:
    """A zero-initialised workspace big enough for this shape, cached per
    device and grown on demand.  The kernels leave its counters at zero, so
    it is reused across calls on one stream; do not share it between
    streams that run GEMMs concurrently."""
    need = qoq_gemm_workspace_bytes(M, N, K, group_size)
    dev = torch.device(device)
    key = dev.index if dev.index is not None else torch.cuda.current_device()
    ws = _ws_cache.get(key)
    if ws is None or ws.numel() < need:
        ws = torch.zeros(max(need, 1 << 20), dtype=torch.uint8, device=dev)
        _ws_cache[key] = ws
    return ws


def qoq_w4a8_gemm(X8: torch.Tensor, s_x: torch.Tensor, packed: PackedWeights,
                  Y: Optional[torch.Tensor] = None, acc_dbg: Optional[torch.Tensor] = None,
                  workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Y fp16 [M, N] = fp16(((float)(X8 . W8hat) * s_x) * s_c)."""
    _need(X8, torch.int8, "X8")
    M, K = X8.shape
    if K != packed.K:
        raise ValueError("K mismatch between X8 and the packed weights")
    N = packed.N
    if Y is None:
        Y = torch.empty(M, N, dtype=torch.float16, device=X8.device)
    if workspace is None:
        workspace = gemm_workspace(max(M, 1), N, K, packed.group_size, X8.device)
    st = lib().qoq_w4a8_gemm(_ptr(X8), _ptr(s_x), _ptr(packed.Wp), _ptr(packed.s_c), _ptr(packed.s_g),
                             _ptr(packed.zs), M, N, K, packed.group_size, _ptr(Y), _ptr(acc_dbg),
                             _ptr(workspace), workspace.numel() * workspace.element_size(),
                             _stream(stream))
    _check("qoq_w4a8_gemm", st)
    return Y


def qoq_w4a8_gemm_fused(X8: torch.Tensor, s_x: torch.Tensor, packed: PackedWeights, epilogue: int,
                        residual: Optional[torch.Tensor] = None, Y: Optional[torch.Tensor] = None,
                        workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """The GEMM with an output-side fusion: QOQ_EPILOGUE_RESIDUAL gives
    fp16(y + residual) ([M, N]); QOQ_EPILOGUE_SILU_MUL (weights from
    qoq_pack_weights_gate_up) gives fp16(silu(gate) * up) ([M, N/2])."""
    _need(X8, torch.int8, "X8")
    M, K = X8.shape
    if K != packed.K:
        raise ValueError("K mismatch between X8 and the packed weights")
    N = packed.N
    if epilogue == QOQ_EPILOGUE_SILU_MUL and not packed.gate_up:
        raise ValueError("the SiLU-gated epilogue needs weights from qoq_pack_weights_gate_up")
    if residual is not None:
        _need(residual, torch.float16, "residual")
    ncol = N // 2 if epilogue == QOQ_EPILOGUE_SILU_MUL else N
    if Y is None:
        Y = torch.empty(M, ncol, dtype=torch.float16, device=X8.device)
    if workspace is None:
        workspace = gemm_workspace(max(M, 1), N, K, packed.group_size, X8.device)
    st = lib().qoq_w4a8_gemm_fused(_ptr(X8), _ptr(s_x), _ptr(packed.Wp), _ptr(packed.s_c), _ptr(packed.s_g),
                                   _ptr(packed.zs), M, N, K, packed.group_size, int(epilogue), _ptr(residual),
                                   _ptr(Y), _ptr(workspace), workspace.numel() * workspace.element_size(),
                                   _stream(stream))
    _check("qoq_w4a8_gemm_fused", st)
    return Y


def qoq_w4a8_gemm_i32(X8: torch.Tensor, packed: PackedWeights, acc: Optional[torch.Tensor] = None,
                      workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """acc int32 [M, N] = X8 . W8hat^T over this call's K (no scales).  X8
    may be a column slice of a wider int8 matrix (row stride passed on)."""
    if not (X8.is_cuda and X8.dtype == torch.int8 and X8.stride(1) == 1):
        raise ValueError("X8 must be a CUDA int8 tensor with unit column stride")
    M, K = X8.shape
    ldx = X8.stride(0) if M > 1 else K
    if K != packed.K:
        raise ValueError("K mismatch between X8 and the packed weights")
    N = packed.N
    if acc is None:
        acc = torch.empty(M, N, dtype=torch.int32, device=X8.device)
    _need(acc, torch.int32, "acc")
    if workspace is None:
        workspace = gemm_workspace(max(M, 1), N, K, packed.group_size, X8.device)
    st = lib().qoq_w4a8_gemm_i32(_ptr(X8), int(ldx), _ptr(packed.Wp), _ptr(packed.s_g), _ptr(packed.zs), M, N, K,
                                 packed.group_size, _ptr(acc), _ptr(workspace),
                                 workspace.numel() * workspace.element_size(), _stream(stream))
    _check("qoq_w4a8_gemm_i32", st)
    return acc


def qoq_epilogue_i32(acc: torch.Tensor, s_x: torch.Tensor, s_c: torch.Tensor, Y: Optional[torch.Tensor] = None,
                     stream=None) -> torch.Tensor:
    """Y fp16 [M, N] = fp16(((float)acc * s_x) * s_c)."""
    _need(acc, torch.int32, "acc")
    M, N = acc.shape
    if Y is None:
        Y = torch.empty(M, N, dtype=torch.float16, device=acc.device)
    st = lib().qoq_epilogue_i32(_ptr(acc), _ptr(s_x), _ptr(s_c), M, N, _ptr(Y), _stream(stream))
    _check("qoq_epilogue_i32", st)
    return Y


def qoq_quantize_weights_w8(W: torch.Tensor, stream=None):
    """W fp32 [N, K] -> (W8 int8 [N, K], s_w int16 [N] FP16 bits): the W8A8 yardstick's weights."""
    _need(W, torch.float32, "W")
    N, K = W.shape
    W8 = torch.empty(N, K, dtype=torch.int8, device=W.device)
    s_w = torch.empty(max(N, 8), dtype=torch.int16, device=W.device)
    st = lib().qoq_quantize_weights_w8(_ptr(W), N, K, _ptr(W8), _ptr(s_w), _stream(stream))
    _check("qoq_quantize_weights_w8", st)
    return W8, s_w


def qoq_w8a8_gemm(X8: torch.Tensor, s_x: torch.Tensor, W8: torch.Tensor, s_w: torch.Tensor,
                  Y: Optional[torch.Tensor] = None, acc_dbg: Optional[torch.Tensor] = None,
                  workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """The W8A8 yardstick: Y fp16 [M, N] = fp16(((float)(X8 . W8^T) * s_x) * s_w)."""
    _need(X8, torch.int8, "X8")
    _need(W8, torch.int8, "W8")
    M, K = X8.shape
    N, K2 = W8.shape
    if K != K2:
        raise ValueError("K mismatch between X8 and W8")
    if Y is None:
        Y = torch.empty(M, N, dtype=torch.float16, device=X8.device)
    if workspace is None:
        workspace = gemm_workspace(max(M, 1), N, K, 128, X8.device)
    st = lib().qoq_w8a8_gemm(_ptr(X8), _ptr(s_x), _ptr(W8), _ptr(s_w), M, N, K, _ptr(Y), _ptr(acc_dbg),
                             _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream))
    _check("qoq_w8a8_gemm", st)
    return Y


def qoq_w4a8_linear(X: torch.Tensor, packed: PackedWeights, X8: Optional[torch.Tensor] = None,
                    s_x: Optional[torch.Tensor] = None, Y: Optional[torch.Tensor] = None,
                    workspace: Optional[torch.Tensor] = None, stream=None):
    """Quantize X (fp16 [M, K]) per token and run the GEMM: the quantizer
    and GEMM kernels back to back, or one launch after
    qoq_set_linear_in_kernel_quant(True) (M <= 148).

    Returns (Y, X8, s_x); bit-identical to qoq_quant_act_per_token followed
    by qoq_w4a8_gemm."""
    _need(X, torch.float16, "X")
    M, K = X.shape
    if K != packed.K:
        raise ValueError("K mismatch between X and the packed weights")
    N = packed.N
    if X8 is None:
        X8 = torch.empty(M, K, dtype=torch.int8, device=X.device)
    if s_x is None:
        s_x = torch.empty(max(M, 8), dtype=torch.int16, device=X.device)
    if Y is None:
        Y = torch.empty(M, N, dtype=torch.float16, device=X.device)
    if workspace is None:
        workspace = gemm_workspace(max(M, 1), N, K, packed.group_size, X.device)
    st = lib().qoq_w4a8_linear(_ptr(X), M, N, K, packed.group_size, _ptr(packed.Wp), _ptr(packed.s_c),
                               _ptr(packed.s_g), _ptr(packed.zs), _ptr(X8), _ptr(s_x), _ptr(Y), _ptr(workspace),
                               workspace.numel() * workspace.element_size(), _stream(stream))
    _check("qoq_w4a8_linear", st)
    return Y, X8, s_x


def qoq_w4a8_gemm_noalloc(X8: torch.Tensor, s_x: torch.Tensor, packed: PackedWeights,
                          Y: torch.Tensor, stream=None) -> torch.Tensor:
    """The GEMM with its scratch in the library's built-in buffer.

    For callers that may not allocate while they run the layer (an engine's
    execute step, a plug-in without an allocator, a real-time path): the
    caller passes a preallocated Y, and the call itself allocates nothing.
    Shapes needing more than QOQ_NOALLOC_SCRATCH_BYTES of scratch raise
    QoQError(QOQ_ERR_SCRATCH_TOO_SMALL); calls that may overlap on the GPU
    must be serialized, since they share the buffer."""
    _need(X8, torch.int8, "X8")
    M, K = X8.shape
    if K != packed.K:
        raise ValueError("K mismatch between X8 and the packed weights")
    st = lib().qoq_w4a8_gemm_noalloc(_ptr(X8), _ptr(s_x), _ptr(packed.Wp), _ptr(packed.s_c),
                                     _ptr(packed.s_g), _ptr(packed.zs), M, packed.N, K,
                                     packed.group_size, _ptr(Y), _stream(stream))
    _check("qoq_w4a8_gemm_noalloc", st)
    return Y


def qoq_dequant_weights_i8(packed: PackedWeights, out: Optional[torch.Tensor] = None,
                           stream=None) -> torch.Tensor:
    if out is None:
        out = torch.empty(packed.N, packed.K, dtype=torch.int8, device=packed.Wp.device)
    st = lib().qoq_dequant_weights_i8(_ptr(packed.Wp), _ptr(packed.s_g), _ptr(packed.zs), packed.N,
                                      packed.K, packed.group_size, _ptr(out), _stream(stream))
    _check("qoq_dequant_weights_i8", st)
    return out


# -------------------------------------------------------- KV4 attention ----
@dataclass
class KV4Cache:
    """A 4-bit KV cache with SmoothAttention factors (layouts of include/qoq.h)."""
    K4: torch.Tensor     # uint8 [B, Hkv, L, d/2]
    V4: torch.Tensor     # uint8 [B, Hkv, L, d/2]
    lam: torch.Tensor    # int16 [B, Hkv, d] FP16 bits
    s_k: torch.Tensor    # int16 [B, Hkv, d] FP16 bits
    s_v: torch.Tensor    # int16 [B, Hkv, d] FP16 bits


def qoq_kv4_cache_quantize(K: torch.Tensor, V: torch.Tensor, stream=None) -> KV4Cache:
    """K, V fp16 [B, Hkv, L, d] -> KV4Cache."""
    _need(K, torch.float16, "K")
    _need(V, torch.float16, "V")
    B, Hkv, L, d = K.shape
    dev = K.device
    c = KV4Cache(torch.empty(B, Hkv, L, d // 2, dtype=torch.uint8, device=dev),
                 torch.empty(B, Hkv, L, d // 2, dtype=torch.uint8, device=dev),
                 torch.empty(B, Hkv, d, dtype=torch.int16, device=dev),
                 torch.empty(B, Hkv, d, dtype=torch.int16, device=dev),
                 torch.empty(B, Hkv, d, dtype=torch.int16, device=dev))
    st = lib().qoq_kv4_cache_quantize(_ptr(K), _ptr(V), B, Hkv, L, d, _ptr(c.K4), _ptr(c.V4), _ptr(c.lam),
                                      _ptr(c.s_k), _ptr(c.s_v), _stream(stream))
    _check("qoq_kv4_cache_quantize", st)
    return c


def qoq_kv4_attention_workspace_bytes(B: int, Hq: int, Hkv: int, L: int, d: int) -> int:
    return int(lib().qoq_kv4_attention_workspace_bytes(int(B), int(Hq), int(Hkv), int(L), int(d)))


def qoq_kv4_decode_attention(q: torch.Tensor, cache: KV4Cache, out: Optional[torch.Tensor] = None,
                             workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """q fp16 [B, Hq, d] -> out fp16 [B, Hq, d]: attention over the KV4 cache."""
    _need(q, torch.float16, "q")
    B, Hq, d = q.shape
    _, Hkv, L, _ = cache.K4.shape
    if out is None:
        out = torch.empty(B, Hq, d, dtype=torch.float16, device=q.device)
    if workspace is None:
        workspace = torch.empty(max(qoq_kv4_attention_workspace_bytes(B, Hq, Hkv, L, d), 16),
                                dtype=torch.uint8, device=q.device)
    st = lib().qoq_kv4_decode_attention(_ptr(q), _ptr(cache.K4), _ptr(cache.V4), _ptr(cache.lam), _ptr(cache.s_k),
                                        _ptr(cache.s_v), B, Hq, Hkv, L, d, _ptr(out), _ptr(workspace),
                                        workspace.numel() * workspace.element_size(), _stream(stream))
    _check("qoq_kv4_decode_attention", st)
    return out


# ---------------------------------------------------------------- layer ----
class W4A8Linear:
    """A linear layer y = x W^T with QoQ W4A8 weights resident on the GPU."""

    def __init__(self, weight_fp32: torch.Tensor, group_size: int = 128):
        W = weight_fp32.to(device="cuda", dtype=torch.float32).contiguous()
        self.packed = qoq_pack_weights(W, group_size)
        self.in_features = W.shape[1]
        self.out_features = W.shape[0]

    def __call__(self, x_fp16: torch.Tensor, stream=None) -> torch.Tensor:
        """y = fp16 W4A8 linear of x (fp16 [M, in_features]) through the layer call."""
        Y, _, _ = qoq_w4a8_linear(x_fp16, self.packed, stream=stream)
        return Y


_HOST_STREAMS = {}
_HOST_STREAMS_LOCK = threading.Lock()


_HOST_CHUNK_BYTES = 16 << 20


def _host_pieces(calls, chunk_rows):
    """The calls cut into row blocks: the layer is row-wise (each output row
    depends on its own input row only, per-token scale included), so a block
    of rows is a call of its own with the same bits.  Blocks of about 16 MB
    of X or Y let one block's copy in overlap the previous block's kernels
    and copy out."""
    out = []
    for x_host, layer, y_host in calls:
        M = x_host.shape[0] if x_host.dim() == 2 else 0
        rows = chunk_rows
        if rows is None:
            width = max(x_host.shape[-1], y_host.shape[-1])
            rows = max(128, _HOST_CHUNK_BYTES // (2 * width) // 128 * 128)
        if M <= rows or y_host.dim() != 2 or y_host.shape[0] != M:
            out.append((x_host, layer, y_host))
            continue
        for r in range(0, M, rows):
            out.append((x_host[r:r + rows], layer, y_host[r:r + rows]))
    return out


def w4a8_linear_host_many(calls, stream=None, chunk_rows: Optional[int] = None) -> list:
    """Several end-to-end calls from host memory, pipelined.  `calls` is a
    list of (x_host, layer, y_host): FP16 X [M][K] in host memory (ideally
    pinned), a W4A8Linear, and a host tensor for Y [M][N] (ideally pinned).
    Each call is cut into blocks of `chunk_rows` token rows (by default about
    16 MB of X or Y per block; the outputs are the same bits).  Block i's copy
    of X to the device, its layer call and its copy of Y back run on three
    streams chained by events, so that one block's copies overlap the other
    blocks' kernels and copies in the other direction (the host link is full
    duplex).  Returns the y_host tensors once all of them hold their results;
    `stream` waits for all of the work, so events on it bracket the whole
    pipeline."""
    if chunk_rows is not None and chunk_rows < 1:
        raise ValueError("chunk_rows must be positive")
    s = stream or torch.cuda.current_stream()
    dev = s.device
    with _HOST_STREAMS_LOCK:
        if dev not in _HOST_STREAMS:
            _HOST_STREAMS[dev] = tuple(torch.cuda.Stream(device=dev) for _ in range(3))
        s_in, s_cmp, s_out = _HOST_STREAMS[dev]
    start = torch.cuda.Event()
    start.record(s)
    for t in (s_in, s_cmp, s_out):
        t.wait_event(start)
    for x_host, layer, y_host in _host_pieces(calls, chunk_rows):
        with torch.cuda.stream(s_in):
            x = x_host.to(dev, non_blocking=True)
        ready = torch.cuda.Event()
        ready.record(s_in)
        s_cmp.wait_event(ready)
        x.record_stream(s_cmp)
        with torch.cuda.stream(s_cmp):
            y = layer(x, stream=s_cmp)
        done = torch.cuda.Event()
        done.record(s_cmp)
        s_out.wait_event(done)
        y.record_stream(s_out)
        with torch.cuda.stream(s_out):
            y_host.copy_(y, non_blocking=True)
    for t in (s_in, s_cmp, s_out):
        e = torch.cuda.Event()
        e.record(t)
        s.wait_event(e)
    s.synchronize()
    return [c[2] for c in calls]


def w4a8_linear_host(x_host: torch.Tensor, layer: W4A8Linear, y_host: Optional[torch.Tensor] = None,
                     stream=None) -> torch.Tensor:
    """End-to-end call from host memory: copy X (fp16, ideally pinned) to the
    device, quantize it, run the GEMM, copy Y back; returns the host Y."""
    s = stream or torch.cuda.current_stream()
    with torch.cuda.stream(s):
        x = x_host.to("cuda", non_blocking=True)
        y = layer(x, stream=s)
        if y_host is None:
            y_host = torch.empty(y.shape, dtype=y.dtype, pin_memory=True)
        y_host.copy_(y, non_blocking=True)
    s.synchronize()
    return y_host
