"""CPU oracle for the QoQ W4A8 linear layer (test infrastructure only).

This package is the independent, slow, plain definition of what the CUDA
library computes.  It is loaded only by the tests, by ``__graft_entry__.smoke``
and by the CPU-baseline leg of ``bench.py``; the library's product path never
imports it, and it imports nothing from the library.

The arithmetic lives in ``qoq_oracle.c`` (plain C, each function citing the
passage of the pages it follows).  This module only marshals numpy arrays in
and out of it with ctypes, and builds the shared object with gcc on first use.

Functions mirror the steps of the layer, in the pages' order:

    quantize_weights  -- stage 1 + stage 2 ("QServe: Low Bit Width Does Not
                         Guarantee High Throughput", section 4, stage-1 and
                         stage-2 equations)
    dequant_weights   -- q*s_g - z*s_g (same section, paragraph after the
                         equations)
    quant_act         -- per-token INT8 ("QServe Guide: W4A8KV4 Quantization
                         for LLM Serving", Deep Dive subsection 1)
    gemm_i32          -- INT32 inner products (QServe Guide, Architecture
                         subsection 2)
    epilogue          -- FP16 output scaling (QServe Guide, Deep Dive
                         subsection 1, output rescaling equation)

Parity of every function here is pinned by tests/test_oracle_*.py against
things other than this code: a hand-worked example, numpy's own binary16
conversion, exhaustive enumeration of the stage-2 group space, exact
big-integer sums, FP64 matmuls and closed forms.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "qoq_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libqoq_oracle.so")
_lock = threading.Lock()
_lib = None

_P = ctypes.c_void_p
_I64 = ctypes.c_int64


def build(force: bool = False) -> str:
    """Compile qoq_oracle.c into libqoq_oracle.so with gcc (no fast-math)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
           "-ffp-contract=off", "-fno-fast-math", "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        lib = ctypes.CDLL(build())
        lib.oracle_half_to_float.argtypes = [ctypes.c_uint16]
        lib.oracle_half_to_float.restype = ctypes.c_float
        lib.oracle_float_to_half_rn.argtypes = [ctypes.c_float]
        lib.oracle_float_to_half_rn.restype = ctypes.c_uint16
        lib.oracle_div_round_half_even.argtypes = [ctypes.c_int, ctypes.c_int]
        lib.oracle_div_round_half_even.restype = ctypes.c_int
        lib.oracle_stage2_group.argtypes = [_P, ctypes.c_int, _P, _P, _P, _P]
        lib.oracle_stage2_group.restype = None
        lib.oracle_quantize_weights.argtypes = [_P, _I64, _I64, _I64, _P, _P, _P, _P, _P, _P]
        lib.oracle_quantize_weights.restype = None
        lib.oracle_dequant_weights.argtypes = [_P, _P, _P, _I64, _I64, _I64, _P]
        lib.oracle_dequant_weights.restype = None
        lib.oracle_quant_act.argtypes = [_P, _I64, _I64, _P, _P]
        lib.oracle_quant_act.restype = None
        lib.oracle_gemm_i32.argtypes = [_P, _P, _I64, _I64, _I64, _P]
        lib.oracle_gemm_i32.restype = None
        lib.oracle_epilogue.argtypes = [_P, _P, _P, _I64, _I64, _P]
        lib.oracle_epilogue.restype = None
        lib.oracle_quantize_weights_w8.argtypes = [_P, _I64, _I64, _P, _P]
        lib.oracle_quantize_weights_w8.restype = None
        lib.oracle_smooth_lambda.argtypes = [_P, _I64, _I64, ctypes.c_double, _P]
        lib.oracle_smooth_lambda.restype = None
        lib.oracle_kv4_quantize.argtypes = [_P, _I64, _I64, _P, _P, _P]
        lib.oracle_kv4_quantize.restype = None
        lib.oracle_kv4_attention.argtypes = [_P, _P, _P, _P, _P, _P, _I64, _I64, _I64, _I64, _P]
        lib.oracle_kv4_attention.restype = None
        lib.oracle_double_to_half_rn.argtypes = [ctypes.c_double]
        lib.oracle_double_to_half_rn.restype = ctypes.c_uint16
        lib.oracle_epilogue_residual.argtypes = [_P, _P, _P, _I64, _I64, _P, _P]
        lib.oracle_epilogue_residual.restype = None
        lib.oracle_epilogue_silu_mul.argtypes = [_P, _P, _P, _I64, _I64, _P]
        lib.oracle_epilogue_silu_mul.restype = None
        lib.oracle_num_threads.argtypes = []
        lib.oracle_num_threads.restype = ctypes.c_int
        lib.oracle_set_num_threads.argtypes = [ctypes.c_int]
        lib.oracle_set_num_threads.restype = None
        _lib = lib
        return lib


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


def num_threads() -> int:
    """OpenMP threads the oracle's parallel loops use."""
    return int(_load().oracle_num_threads())


def set_num_threads(n: int) -> None:
    """Sets the OpenMP threads of later calls from this thread (timing only:
    the results do not depend on it)."""
    _load().oracle_set_num_threads(int(n))


# ---------------------------------------------------------------- fp16 ----
def half_to_float(bits: int) -> float:
    return float(_load().oracle_half_to_float(int(bits)))


def float_to_half_bits(x: float) -> int:
    return int(_load().oracle_float_to_half_rn(float(np.float32(x))))


def half_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Vector widening through the oracle's own binary16 decoder."""
    lib = _load()
    flat = np.ascontiguousarray(bits, dtype=np.uint16).ravel()
    out = np.fromiter((lib.oracle_half_to_float(int(b)) for b in flat),
                      dtype=np.float32, count=flat.size)
    return out.reshape(np.shape(bits))


def f32_to_half_bits(x: np.ndarray) -> np.ndarray:
    """Vector narrowing through the oracle's own binary16 encoder."""
    lib = _load()
    flat = np.ascontiguousarray(x, dtype=np.float32).ravel()
    out = np.fromiter((lib.oracle_float_to_half_rn(float(v)) for v in flat),
                      dtype=np.uint16, count=flat.size)
    return out.reshape(np.shape(x))


def div_round_half_even(a: int, b: int) -> int:
    return int(_load().oracle_div_round_half_even(int(a), int(b)))


# ------------------------------------------------------------- stage 2 ----
def stage2_group(w8: np.ndarray):
    """Stage 2 on one group of INT8 values -> (q, s_g, z, zs)."""
    w8 = np.ascontiguousarray(w8, dtype=np.int8)
    q = np.zeros(w8.size, dtype=np.uint8)
    sg = np.zeros(1, np.uint8)
    z = np.zeros(1, np.uint8)
    zs = np.zeros(1, np.uint8)
    _load().oracle_stage2_group(_ptr(w8), int(w8.size), _ptr(q), _ptr(sg), _ptr(z), _ptr(zs))
    return q, int(sg[0]), int(z[0]), int(zs[0])


# ------------------------------------------------------------- weights ----
def quantize_weights(W: np.ndarray, group_size: int) -> dict:
    """Stages 1 + 2 of progressive group quantization.

    W: float32 [N][K] (row n = output channel).  group_size must divide K.
    Returns canonical row-major arrays: s_c (uint16 FP16 bits [N]),
    W8 (int8 [N][K]), q (uint8 [N][K], values 0..15), s_g, z, zs
    (uint8 [N][K/G]).
    """
    W = np.ascontiguousarray(W, dtype=np.float32)
    N, K = W.shape
    G = int(group_size)
    if G <= 0 or K % G:
        raise ValueError("group_size must divide K")
    ng = K // G
    out = dict(
        s_c=np.zeros(N, np.uint16), W8=np.zeros((N, K), np.int8), q=np.zeros((N, K), np.uint8),
        s_g=np.zeros((N, ng), np.uint8), z=np.zeros((N, ng), np.uint8), zs=np.zeros((N, ng), np.uint8))
    _load().oracle_quantize_weights(_ptr(W), N, K, G, _ptr(out["s_c"]), _ptr(out["W8"]),
                                    _ptr(out["q"]), _ptr(out["s_g"]), _ptr(out["z"]), _ptr(out["zs"]))
    return out


def dequant_weights(q: np.ndarray, s_g: np.ndarray, zs: np.ndarray, group_size: int) -> np.ndarray:
    """W8hat[n][k] = q*s_g - zs, int8 [N][K]."""
    q = np.ascontiguousarray(q, np.uint8)
    s_g = np.ascontiguousarray(s_g, np.uint8)
    zs = np.ascontiguousarray(zs, np.uint8)
    N, K = q.shape
    out = np.zeros((N, K), np.int8)
    _load().oracle_dequant_weights(_ptr(q), _ptr(s_g), _ptr(zs), N, K, int(group_size), _ptr(out))
    return out


# ---------------------------------------------------------- activations ----
def quant_act(X_half: np.ndarray):
    """Per-token INT8: X (float16 or uint16 FP16 bits [M][K]) -> (X8 int8, s_x uint16 bits)."""
    X = np.ascontiguousarray(X_half)
    if X.dtype == np.float16:
        X = X.view(np.uint16)
    X = np.ascontiguousarray(X, np.uint16)
    M, K = X.shape
    X8 = np.zeros((M, K), np.int8)
    s_x = np.zeros(M, np.uint16)
    _load().oracle_quant_act(_ptr(X), M, K, _ptr(X8), _ptr(s_x))
    return X8, s_x


# ------------------------------------------------------------ GEMM ----
def gemm_i32(X8: np.ndarray, W8hat: np.ndarray) -> np.ndarray:
    """acc[m][n] = sum_k X8[m][k] * W8hat[n][k] (int32)."""
    X8 = np.ascontiguousarray(X8, np.int8)
    W8hat = np.ascontiguousarray(W8hat, np.int8)
    M, K = X8.shape
    N, K2 = W8hat.shape
    if K != K2:
        raise ValueError("K mismatch")
    acc = np.zeros((M, N), np.int32)
    _load().oracle_gemm_i32(_ptr(X8), _ptr(W8hat), M, N, K, _ptr(acc))
    return acc


def epilogue(acc: np.ndarray, s_x: np.ndarray, s_c: np.ndarray) -> np.ndarray:
    """Y = fp16_rn(((float)acc * sx) * sc) -> uint16 FP16 bits [M][N]."""
    acc = np.ascontiguousarray(acc, np.int32)
    s_x = np.ascontiguousarray(s_x, np.uint16)
    s_c = np.ascontiguousarray(s_c, np.uint16)
    M, N = acc.shape
    Y = np.zeros((M, N), np.uint16)
    _load().oracle_epilogue(_ptr(acc), _ptr(s_x), _ptr(s_c), M, N, _ptr(Y))
    return Y


def double_to_half_bits(x: float) -> int:
    return int(_load().oracle_double_to_half_rn(float(x)))


def epilogue_residual(acc: np.ndarray, s_x: np.ndarray, s_c: np.ndarray, R: np.ndarray) -> np.ndarray:
    """Y = fp16_rn((float)y + (float)R), y the layer's FP16 output -> uint16 bits [M][N]."""
    acc = np.ascontiguousarray(acc, np.int32)
    s_x = np.ascontiguousarray(s_x, np.uint16)
    s_c = np.ascontiguousarray(s_c, np.uint16)
    R = np.ascontiguousarray(R)
    if R.dtype == np.float16:
        R = R.view(np.uint16)
    R = np.ascontiguousarray(R, np.uint16)
    M, N = acc.shape
    Y = np.zeros((M, N), np.uint16)
    _load().oracle_epilogue_residual(_ptr(acc), _ptr(s_x), _ptr(s_c), M, N, _ptr(R), _ptr(Y))
    return Y


def epilogue_silu_mul(acc: np.ndarray, s_x: np.ndarray, s_c: np.ndarray) -> np.ndarray:
    """Out[m][j] = fp16_rn(silu(g) * u) with g, u the FP16 outputs of gate column j
    and up column I + j (acc has 2I columns) -> uint16 bits [M][I]."""
    acc = np.ascontiguousarray(acc, np.int32)
    s_x = np.ascontiguousarray(s_x, np.uint16)
    s_c = np.ascontiguousarray(s_c, np.uint16)
    M, N2 = acc.shape
    if N2 % 2:
        raise ValueError("the gate/up pair needs an even number of columns")
    Out = np.zeros((M, N2 // 2), np.uint16)
    _load().oracle_epilogue_silu_mul(_ptr(acc), _ptr(s_x), _ptr(s_c), M, N2, _ptr(Out))
    return Out


def quantize_weights_w8(W: np.ndarray):
    """The W8A8 yardstick's weights: (W8 int8 [N][K], s_w uint16 FP16 bits [N])."""
    W = np.ascontiguousarray(W, dtype=np.float32)
    N, K = W.shape
    W8 = np.zeros((N, K), np.int8)
    s_w = np.zeros(N, np.uint16)
    _load().oracle_quantize_weights_w8(_ptr(W), N, K, _ptr(s_w), _ptr(W8))
    return W8, s_w


def linear_w8a8(X_half: np.ndarray, W: np.ndarray) -> dict:
    """The W8A8 yardstick layer on the CPU."""
    W8, s_w = quantize_weights_w8(W)
    X8, s_x = quant_act(X_half)
    acc = gemm_i32(X8, W8)
    Y = epilogue(acc, s_x, s_w)
    return dict(W8=W8, s_w=s_w, X8=X8, s_x=s_x, acc=acc, Y=Y)


# ---------------------------------------------------- KV4 attention ----
def _bits16(x):
    x = np.ascontiguousarray(x)
    if x.dtype == np.float16:
        x = x.view(np.uint16)
    return np.ascontiguousarray(x, np.uint16)


def smooth_lambda(K: np.ndarray, alpha: float = 0.5) -> np.ndarray:
    """SmoothAttention factors of one KV head: K [L][d] FP16 -> lambda [d] FP16 bits."""
    K = _bits16(K)
    L, d = K.shape
    lam = np.zeros(d, np.uint16)
    _load().oracle_smooth_lambda(_ptr(K), L, d, float(alpha), _ptr(lam))
    return lam


def kv4_quantize(X: np.ndarray, lam: np.ndarray = None):
    """X [L][d] FP16 -> (codes int8 [L][d] in -8..7, s uint16 FP16 bits [d]); with lam,
    X is divided by it first (the smoothed keys)."""
    X = _bits16(X)
    L, d = X.shape
    codes = np.zeros((L, d), np.int8)
    s = np.zeros(d, np.uint16)
    lp = None if lam is None else _bits16(lam)
    _load().oracle_kv4_quantize(_ptr(X), L, d, None if lp is None else _ptr(lp), _ptr(codes), _ptr(s))
    return codes, s


def kv4_attention(q: np.ndarray, k_codes: np.ndarray, s_k: np.ndarray, v_codes: np.ndarray,
                  s_v: np.ndarray, lam: np.ndarray) -> np.ndarray:
    """One sequence: q [Hq][d] FP16; codes [Hkv][L][d]; s_k, s_v, lam [Hkv][d] FP16 bits.
    Returns out [Hq][d] FP16 bits."""
    q = _bits16(q)
    Hq, d = q.shape
    Hkv, L, d2 = k_codes.shape
    assert d2 == d and Hq % Hkv == 0
    out = np.zeros((Hq, d), np.uint16)
    _load().oracle_kv4_attention(_ptr(q), _ptr(np.ascontiguousarray(k_codes, np.int8)), _ptr(_bits16(s_k)),
                                 _ptr(np.ascontiguousarray(v_codes, np.int8)), _ptr(_bits16(s_v)),
                                 _ptr(_bits16(lam)), Hq, Hkv, L, d, _ptr(out))
    return out


def kv4_decode(q: np.ndarray, K: np.ndarray, V: np.ndarray, alpha: float = 0.5) -> dict:
    """The whole KV4 step for one sequence on the CPU: q [Hq][d], K, V [Hkv][L][d] FP16."""
    Hkv, L, d = K.shape
    lam = np.stack([smooth_lambda(K[g], alpha) for g in range(Hkv)])
    kq = [kv4_quantize(K[g], lam[g]) for g in range(Hkv)]
    vq = [kv4_quantize(V[g]) for g in range(Hkv)]
    k_codes = np.stack([c for c, _ in kq]); s_k = np.stack([s for _, s in kq])
    v_codes = np.stack([c for c, _ in vq]); s_v = np.stack([s for _, s in vq])
    out = kv4_attention(q, k_codes, s_k, v_codes, s_v, lam)
    return dict(lam=lam, k_codes=k_codes, s_k=s_k, v_codes=v_codes, s_v=s_v, out=out)


# ------------------------------------------------------------ chains ----
def linear(X_half: np.ndarray, W: np.ndarray, group_size: int) -> dict:
    """The whole layer on the CPU: every intermediate, canonical layouts."""
    wq = quantize_weights(W, group_size)
    W8hat = dequant_weights(wq["q"], wq["s_g"], wq["zs"], group_size)
    X8, s_x = quant_act(X_half)
    acc = gemm_i32(X8, W8hat)
    Y = epilogue(acc, s_x, wq["s_c"])
    return dict(wq, W8hat=W8hat, X8=X8, s_x=s_x, acc=acc, Y=Y)


def linear_sampled(X_half: np.ndarray, W: np.ndarray, group_size: int,
                   rows: np.ndarray, cols: np.ndarray) -> dict:
    """Outputs Y[rows][:, cols] only.

    Weight quantization is per output channel and activation quantization is
    per token, so quantizing only the sampled channels and tokens gives the
    same values as the full computation at those positions.
    """
    rows = np.asarray(rows, np.int64)
    cols = np.asarray(cols, np.int64)
    Xs = np.ascontiguousarray(np.asarray(X_half)[rows])
    Ws = np.ascontiguousarray(np.asarray(W, np.float32)[cols])
    return linear(Xs, Ws, group_size)
