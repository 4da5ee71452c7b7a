"""The C ABI without a GPU: the library loads, exports exactly what
include/qoq.h declares, and its host-side checks reject bad arguments
before touching any device."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "qoq.h")


@pytest.fixture(scope="module")
def L():
    from w4a8_integer_gemm_b200 import build_lib
    build_lib.build()
    import w4a8_integer_gemm_b200 as q
    return q.lib()


def declared():
    txt = open(HEADER).read()
    return set(re.findall(r"QOQ_API\s+[\w\s\*]+?\b(qoq_\w+)\s*\(", txt))


def test_exports_every_declared_symbol(L):
    import w4a8_integer_gemm_b200 as q
    names = declared()
    assert len(names) == 26
    for n in names:
        assert hasattr(L, n), n
    assert names == set(q.SIGNATURES)
    # nothing else with C linkage is exported
    out = os.popen(f"nm -D --defined-only {q.LIB_PATH}").read().split("\n")
    exported = {l.split()[-1] for l in out if l.strip() and l.split()[-1].startswith("qoq_")}
    assert exported == names


def test_status_strings(L):
    import w4a8_integer_gemm_b200 as q
    for s in (0, -1, -2, -3, -4, -5):
        assert len(q.qoq_status_string(s)) >= 2
    assert q.qoq_status_string(7) == "unknown status"


def test_size_queries(L):
    import w4a8_integer_gemm_b200 as q
    # codes, plus the tables the chunks carry for 128-wide groups
    assert q.qoq_packed_weight_bytes(14336, 4096, 4096) == 14336 * 4096 // 2
    assert q.qoq_packed_weight_bytes(14336, 4096, 128) == 14336 * 4096 // 2 + 14336 * 4096 // 64
    assert q.qoq_packed_weight_bytes(100, 4096, 128) == 0
    assert q.qoq_packed_weight_bytes(128, 100, 100) == 0
    assert q.qoq_packed_weight_bytes(128, 512, 64) == 0
    assert q.qoq_gemm_workspace_bytes(1, 14336, 4096, 128) > 0
    assert q.qoq_gemm_workspace_bytes(1, 14336, 4096, 64) == 0      # group size not supported
    assert q.qoq_gemm_workspace_bytes(0, 512, 512, 128) == 0
    # 8192 bytes of counters, then for each of <= 148 CTAs one partial tile
    # of BN=16 tokens x 128 channels x int32
    assert q.qoq_gemm_workspace_bytes(1, 14336, 4096, 128) == 8192 + 148 * 16 * 128 * 4
    # grid = units when there are fewer units than SMs (4 tiles x 4 K blocks of 128,
    # the narrowest stage any configuration uses)
    assert q.qoq_gemm_workspace_bytes(1, 512, 512, 128) == 8192 + 16 * 16 * 128 * 4
    # 256-token tiles use 128-wide K blocks: 4 m-tiles x 64 n-tiles x 64 blocks -> 148 CTAs
    assert q.qoq_gemm_workspace_bytes(1024, 8192, 8192, 128) == 8192 + 148 * 256 * 128 * 4
    # Few tiles: the default rule narrows M = 256, N = K = 4096 to 64-token tiles, but the
    # workspace also covers the 256-token tiles of the other rule (148 CTAs either way).
    assert q.qoq_gemm_workspace_bytes(256, 4096, 4096, 128) == 8192 + 148 * 256 * 128 * 4
    # M = 200, N = 512, K = 1024: 64-token tiles give 4 x 4 tiles x 8 K blocks of 128 = 128
    # units, 256-token tiles 4 tiles x 8 K blocks = 32: 128 CTAs, 256-token slots.
    assert q.qoq_gemm_workspace_bytes(200, 512, 1024, 128) == 8192 + 128 * 256 * 128 * 4
    # and the size does not depend on the switch
    sizes = []
    for narrow in (False, True):
        q.qoq_set_gemm_narrow_tiles(narrow)
        sizes.append(q.qoq_gemm_workspace_bytes(200, 512, 1024, 128))
    assert sizes[0] == sizes[1]


def _fake(addr):
    return ctypes.c_void_p(addr)


def test_invalid_arguments_rejected_on_host(L):
    A = _fake(0x10000)          # aligned, never dereferenced: checks fail first
    B = _fake(0x10001)          # misaligned
    INVALID = -1
    g = L.qoq_w4a8_gemm
    ok_args = [A] * 6 + [16, 512, 512, 128, A, None, A, 1 << 30, None]

    def call(**kw):
        a = list(ok_args)
        names = ["X8", "s_x", "Wp", "s_c", "s_g", "zs", "M", "N", "K", "G", "Y", "acc", "ws", "wsb", "st"]
        for k, v in kw.items():
            a[names.index(k)] = v
        return g(*a)

    assert call(K=500) == INVALID
    assert call(K=0) == INVALID
    assert call(N=500) == INVALID
    assert call(G=64) == INVALID
    assert call(M=-1) == INVALID
    assert call(X8=B) == INVALID
    assert call(Y=None) == INVALID
    assert call(ws=None) == INVALID
    assert call(wsb=16) == INVALID
    assert call(acc=B) == INVALID
    assert call(M=0) == 0                        # empty problem: nothing to do
    assert L.qoq_quant_act_per_token(A, 4, 100, A, A, None, None) == INVALID
    assert L.qoq_quant_act_per_token(A, 0, 512, A, A, None, None) == 0
    assert L.qoq_quant_act_per_token(A, 4, 512, A, A, _fake(0x10002), None) == INVALID   # rowsum misaligned
    assert L.qoq_pack_weights(A, 512, 512, 100, A, A, A, A, None, None, None) == INVALID
    assert L.qoq_pack_weights(B, 512, 512, 128, A, A, A, A, None, None, None) == INVALID
    assert L.qoq_pack_weights(A, 512, 512, 128, A, A, A, A, None, B, None) == INVALID     # q_dbg misaligned
    assert L.qoq_dequant_weights_i8(A, A, A, 512, 512, 3, A, None) == INVALID
    assert L.qoq_set_gemm_a_in_tmem(2) == INVALID
    assert L.qoq_set_gemm_cta_pairs(2) == INVALID
    assert L.qoq_set_gemm_narrow_tiles(-1) == INVALID
    assert L.qoq_set_gemm_half_ctas(3) == INVALID
    assert L.qoq_set_gemm_gemv(2) == INVALID
    assert L.qoq_set_linear_in_kernel_quant(2) == INVALID
    assert L.qoq_selftest_wait_timeout(ctypes.c_ulonglong(10), None) == INVALID          # budget too short
    assert L.qoq_selftest_wait_timeout(ctypes.c_ulonglong(10 ** 12), None) == INVALID    # too long
    # the fused layer call: X, M, N, K, G, Wp, s_c, s_g, zs, X8, s_x, Y, ws, wsb, stream
    f = L.qoq_w4a8_linear
    fused_ok = [A, 16, 512, 512, 128, A, A, A, A, A, A, A, A, 1 << 30, None]

    def fcall(i, v):
        a = list(fused_ok)
        a[i] = v
        return f(*a)

    assert fcall(0, B) == INVALID                 # misaligned X
    assert fcall(0, None) == INVALID
    assert fcall(3, 500) == INVALID               # K
    assert fcall(4, 64) == INVALID                # group size
    assert fcall(9, None) == INVALID              # X8
    assert fcall(10, B) == INVALID                # s_x
    assert fcall(13, 16) == INVALID               # workspace too small
    assert fcall(1, 0) == 0                       # M = 0: nothing to do


def test_noalloc_scratch_bound_and_checks(L):
    """The no-alloc entry point: its built-in buffer holds the scratch of
    every shape up to 128 tokens (the header's promise), and it applies the
    same host-side checks as qoq_w4a8_gemm before touching any device."""
    import w4a8_integer_gemm_b200 as q
    for N in (128, 4096, 1 << 20):
        for K in (128, 4096, 65536):
            for G in (128, K):
                for M in (1, 16, 64, 65, 128):
                    assert 0 < q.qoq_gemm_workspace_bytes(M, N, K, G) <= q.QOQ_NOALLOC_SCRATCH_BYTES, (M, N, K, G)
    A = _fake(0x10000)
    B = _fake(0x10001)
    INVALID = -1
    f = L.qoq_w4a8_gemm_noalloc
    ok = [A] * 6 + [16, 512, 512, 128, A, None]

    def call(i, v):
        a = list(ok)
        a[i] = v
        return f(*a)

    for i in range(6):
        assert call(i, None) == INVALID          # each input pointer null
        assert call(i, B) == INVALID             # each input pointer misaligned
    assert call(10, None) == INVALID             # Y
    assert call(10, B) == INVALID
    assert call(9, 64) == INVALID                # group size neither 128 nor K
    assert call(9, 256) == INVALID
    assert call(8, 500) == INVALID               # K
    assert call(7, 500) == INVALID               # N
    assert call(6, -1) == INVALID                # M
    assert call(6, 0) == 0                       # empty problem
