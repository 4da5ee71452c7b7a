"""Parity of the CUDA path against the CPU oracle, through the C ABI.

Bit-exact: packed codes, group tables, channel and token scales, INT8
activations, INT8 dequantized weights, INT32 accumulators.  FP16 outputs:
|err| <= 1 FP16 ulp of the oracle value (the kernel rounds in the oracle's
order, so in practice they are equal).
"""
import numpy as np
import pytest
import torch

import oracle
import w4a8_integer_gemm_b200 as q
from w4a8_integer_gemm_b200 import workloads as wl
from layout_ref import pack_reference, tables_reference

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from w4a8_integer_gemm_b200 import build_lib
    build_lib.build()
    q.lib()
    yield
    q.qoq_set_gemm_a_in_tmem(True)


def _u16(t):
    return t.cpu().view(torch.int16).numpy().view(np.uint16)


def assert_half_within_1ulp(got_bits, ref_bits):
    g = got_bits.view(np.float16).astype(np.float64)
    r = ref_bits.view(np.float16).astype(np.float64)
    ulp = np.spacing(np.abs(r).astype(np.float16)).astype(np.float64)
    bad = np.abs(g - r) > ulp
    assert not bad.any(), f"{bad.sum()} outputs beyond 1 ulp, first at {np.argwhere(bad)[:5].tolist()}"


def run_layer(X, W, G, a_in_tmem=True, with_acc=True):
    q.qoq_set_gemm_a_in_tmem(a_in_tmem)
    Xd = X.cuda()
    Wd = W.cuda()
    packed = q.qoq_pack_weights(Wd, G)
    X8, s_x = q.qoq_quant_act_per_token(Xd)
    M, N = X.shape[0], W.shape[0]
    acc = torch.full((M, N), -7, dtype=torch.int32, device="cuda") if with_acc else None
    Y = q.qoq_w4a8_gemm(X8, s_x, packed, acc_dbg=acc)
    torch.cuda.synchronize()
    assert q.qoq_device_error() == q.QOQ_OK
    return packed, X8, s_x, Y, acc


# ------------------------------------------------------- activations ----
@pytest.mark.parametrize("M,K", [(1, 128), (16, 512), (33, 4096), (5, 24576), (3, 32768)])
def test_act_quant_bit_exact(M, K):
    X = wl.make_activations(M, K, wl.LLAMA, seed=100 + M)
    X8, s_x = q.qoq_quant_act_per_token(X.cuda())
    rX8, rs = oracle.quant_act(X.numpy())
    assert np.array_equal(X8.cpu().numpy(), rX8)
    assert np.array_equal(_u16(s_x)[:M], rs)


@pytest.mark.parametrize("M,K", [(1, 128), (16, 512), (33, 4096), (5, 24576)])
def test_act_quant_rowsum_exact(M, K):
    """The optional rowsum output equals the sum of the oracle's INT8 row."""
    X = wl.make_activations(M, K, wl.LLAMA, seed=150 + M)
    rowsum = torch.full((M,), 12345, dtype=torch.int32, device="cuda")
    X8, s_x = q.qoq_quant_act_per_token(X.cuda(), rowsum=rowsum)
    rX8, rs = oracle.quant_act(X.numpy())
    assert np.array_equal(X8.cpu().numpy(), rX8)
    assert np.array_equal(rowsum.cpu().numpy(), rX8.astype(np.int64).sum(axis=1))


def test_act_quant_degenerate_rows():
    X = torch.zeros(4, 256, dtype=torch.float16)
    X[1, :] = 6e-8
    X[2, 0], X[2, 1] = 1e-4, -1e-4
    X[3, :] = torch.linspace(-3, 3, 256).half()
    X8, s_x = q.qoq_quant_act_per_token(X.cuda())
    rX8, rs = oracle.quant_act(X.numpy())
    assert np.array_equal(X8.cpu().numpy(), rX8)
    assert np.array_equal(_u16(s_x)[:4], rs)


def _boundary_rows(K):
    """Rows whose values sit on and next to the rounding boundaries of the
    INT8 grid: x near (k + 1/2) * s_x for k = -127 .. 126 and their FP16
    neighbours up to 3 ulps away, with max |x| fixed by element 0 (several
    row maxima, among them ones that make s_x a power of two, so that the
    ties are exact)."""
    rows = []
    for A in (127.0, 63.5, 1.0, 3.3, 0.0137, 1000.0, 17.25):
        sx = float(np.float16(np.float32(A) / np.float32(127.0)))
        vals = []
        for k in range(-127, 127):
            v = np.float16((k + 0.5) * sx)
            lo = hi = v
            vals.append(v)
            for _ in range(3):
                lo = np.nextafter(lo, np.float16(-np.inf))
                hi = np.nextafter(hi, np.float16(np.inf))
                vals += [lo, hi]
        row = np.resize(np.array(vals, dtype=np.float16), K)
        row[0] = np.float16(A) if A < 65504 else row[0]
        rows.append(row)
    return np.stack(rows)


@pytest.mark.parametrize("K", [2048, 8192, 24576])
def test_act_quant_rounding_boundaries(K):
    """Values within a few ulps of x / s_x = k + 1/2: the quantizer's
    reciprocal shortcut must round them exactly as the IEEE division does."""
    X = torch.from_numpy(_boundary_rows(K))
    X8, s_x = q.qoq_quant_act_per_token(X.cuda())
    rX8, rs = oracle.quant_act(X.numpy())
    assert np.array_equal(_u16(s_x)[:X.shape[0]], rs)
    assert np.array_equal(X8.cpu().numpy(), rX8)


# ----------------------------------------------------------- packing ----
@pytest.mark.parametrize("N,K,G", [(128, 128, 128), (512, 512, 128), (512, 512, 512), (384, 4096, 128),
                                   (256, 4096, 4096)])
def test_pack_bit_exact(N, K, G):
    W = wl.make_weights(N, K, wl.LLAMA, seed=200 + N + K)
    p = q.qoq_pack_weights(W.cuda(), G)
    r = oracle.quantize_weights(W.numpy(), G)
    assert np.array_equal(_u16(p.s_c), r["s_c"])
    assert np.array_equal(p.s_g.cpu().numpy(), tables_reference(r["s_g"]))
    assert np.array_equal(p.zs.cpu().numpy(), tables_reference(r["zs"]))
    assert np.array_equal(p.Wp.cpu().numpy(), pack_reference(r["q"], G, r["s_g"], r["zs"]))


@pytest.mark.parametrize("N,K,G", [(128, 128, 128), (384, 4096, 128), (256, 1024, 1024)])
def test_pack_debug_outputs_exact(N, K, G):
    """The optional canonical codes and zero points equal the oracle's."""
    W = wl.make_weights(N, K, wl.LLAMA, seed=250 + N + K)
    z_dbg = torch.full((N, K // G), 99, dtype=torch.uint8, device="cuda")
    q_dbg = torch.full((N, K), 99, dtype=torch.uint8, device="cuda")
    p = q.qoq_pack_weights(W.cuda(), G, z_dbg=z_dbg, q_dbg=q_dbg)
    r = oracle.quantize_weights(W.numpy(), G)
    assert np.array_equal(q_dbg.cpu().numpy(), r["q"])
    assert np.array_equal(z_dbg.cpu().numpy(), r["z"])
    # the tables written beside them are unchanged by the extra outputs
    assert np.array_equal(p.Wp.cpu().numpy(), pack_reference(r["q"], G, r["s_g"], r["zs"]))


def test_pack_degenerate_rows():
    W = torch.zeros(128, 256)
    W[1, 5] = 1e-9
    W[2, :] = 1e-5
    W[3, :] = torch.linspace(-2, 2, 256)
    W[4, ::2] = 1.0
    p = q.qoq_pack_weights(W.cuda(), 128)
    r = oracle.quantize_weights(W.numpy(), 128)
    assert np.array_equal(_u16(p.s_c), r["s_c"])
    assert np.array_equal(p.s_g.cpu().numpy(), tables_reference(r["s_g"]))
    assert np.array_equal(p.zs.cpu().numpy(), tables_reference(r["zs"]))
    assert np.array_equal(p.Wp.cpu().numpy(), pack_reference(r["q"], 128, r["s_g"], r["zs"]))


@pytest.mark.parametrize("N,K,G", [(512, 512, 128), (256, 1024, 1024)])
def test_dequant_bit_exact(N, K, G):
    W = wl.make_weights(N, K, wl.QWEN, seed=300 + K)
    p = q.qoq_pack_weights(W.cuda(), G)
    W8hat = q.qoq_dequant_weights_i8(p).cpu().numpy()
    r = oracle.quantize_weights(W.numpy(), G)
    ref = oracle.dequant_weights(r["q"], r["s_g"], r["zs"], G)
    assert np.array_equal(W8hat, ref)
    assert np.abs(W8hat.astype(int)).max() <= 127


# -------------------------------------------------------------- GEMM ----
GEMM_CASES = [
    # M spans every token-tile width (16/32/64/128/256) and ragged tails
    (1, 512, 512, 128), (7, 512, 512, 512), (16, 512, 512, 128), (17, 1024, 384, 128),
    (33, 512, 640, 128), (64, 1024, 512, 1024), (100, 512, 256, 128), (128, 512, 512, 128),
    (200, 768, 512, 128), (256, 512, 384, 512), (300, 1024, 640, 128), (513, 512, 256, 128),
]


@pytest.mark.parametrize("narrow", [True, False], ids=["narrow", "wide"])
@pytest.mark.parametrize("a_in_tmem", [False, True], ids=["A_smem", "A_tmem"])
@pytest.mark.parametrize("M,K,N,G", GEMM_CASES)
def test_gemm_bit_exact(M, K, N, G, a_in_tmem, narrow):
    # narrow=False keeps the 128/256-token tiles that the default rule
    # replaces with 64-token ones at these small N
    X = wl.make_activations(M, K, wl.LLAMA, seed=400 + M)
    W = wl.make_weights(N, K, wl.LLAMA, seed=500 + N + K)
    q.qoq_set_gemm_narrow_tiles(narrow)
    try:
        _, X8, s_x, Y, acc = run_layer(X, W, G, a_in_tmem)
    finally:
        q.qoq_set_gemm_narrow_tiles(True)
    r = oracle.linear(X.numpy(), W.numpy(), G)
    assert np.array_equal(acc.cpu().numpy(), r["acc"])
    assert_half_within_1ulp(_u16(Y), r["Y"])


HALF_CASES = [c for c in GEMM_CASES if c[0] <= 64] + [(1, 4096, 1024, 128), (64, 4096, 2048, 4096),
                                                   (40, 8192, 1024, 128), (3, 24576, 256, 128)]


@pytest.mark.parametrize("M,K,N,G", HALF_CASES)
def test_gemm_bit_exact_half_ctas(M, K, N, G):
    """Token tiles up to 64 in half-SM CTAs (two per SM): INT32 exact."""
    X = wl.make_activations(M, K, wl.LLAMA, seed=410 + M)
    W = wl.make_weights(N, K, wl.LLAMA, seed=510 + N + K)
    q.qoq_set_gemm_half_ctas(True)
    q.qoq_set_gemm_gemv(False)   # M <= 8 would otherwise take the decode kernel
    try:
        _, X8, s_x, Y, acc = run_layer(X, W, G, True)
        # several launches in a row on the stream: CTAs of consecutive GEMMs
        # share SMs
        packed = q.qoq_pack_weights(W.cuda(), G)
        outs = []
        for _ in range(6):
            a2 = torch.zeros_like(acc)
            outs.append((q.qoq_w4a8_gemm(X8, s_x, packed, acc_dbg=a2), a2))
        torch.cuda.synchronize()
        assert q.qoq_device_error() == q.QOQ_OK
    finally:
        q.qoq_set_gemm_half_ctas(False)
        q.qoq_set_gemm_gemv(True)
    r = oracle.linear(X.numpy(), W.numpy(), G)
    assert np.array_equal(acc.cpu().numpy(), r["acc"])
    assert_half_within_1ulp(_u16(Y), r["Y"])
    for Yi, ai in outs:
        assert torch.equal(ai, acc) and torch.equal(Yi.view(torch.int16), Y.view(torch.int16))


def test_tiny_workload_full_parity():
    """16 x 512 x 512, g128, the tiny workload's distribution and seeds."""
    w = wl.WORKLOADS["tiny"]
    X, W = wl.make_case(w, 0)
    s = w.shapes[0]
    packed, X8, s_x, Y, acc = run_layer(X, W, s.G)
    r = oracle.linear(X.numpy(), W.numpy(), s.G)
    assert np.array_equal(packed.Wp.cpu().numpy(), pack_reference(r["q"], s.G, r["s_g"], r["zs"]))
    assert np.array_equal(X8.cpu().numpy(), r["X8"])
    assert np.array_equal(acc.cpu().numpy(), r["acc"])
    assert np.array_equal(q.qoq_dequant_weights_i8(packed).cpu().numpy(), r["W8hat"])
    assert_half_within_1ulp(_u16(Y), r["Y"])


def test_repeated_calls_reuse_workspace():
    """Split tiles leave the workspace counters at zero: back-to-back calls
    (and a call with a different shape in between) give identical results."""
    X = wl.make_activations(8, 4096, wl.LLAMA, seed=61)
    W = wl.make_weights(1024, 4096, wl.LLAMA, seed=62)
    packed, X8, s_x, Y1, acc1 = run_layer(X, W, 128)
    X2 = wl.make_activations(40, 4096, wl.LLAMA, seed=63)
    X82, s_x2 = q.qoq_quant_act_per_token(X2.cuda())
    q.qoq_w4a8_gemm(X82, s_x2, packed)
    for _ in range(3):
        acc = torch.zeros_like(acc1)
        Y = q.qoq_w4a8_gemm(X8, s_x, packed, acc_dbg=acc)
        assert torch.equal(acc, acc1) and torch.equal(Y, Y1)
    assert q.qoq_device_error() == q.QOQ_OK


def test_one_workspace_across_shapes():
    """The same (cached) workspace serves shapes with different token tiles
    and split layouts in any order."""
    seq = [(200, 512, 384, 128), (1, 512, 512, 128), (64, 1024, 512, 1024), (16, 512, 256, 128),
           (300, 1024, 640, 128), (1, 512, 512, 128)]
    for i, (M, K, N, G) in enumerate(seq):
        X = wl.make_activations(M, K, wl.LLAMA, seed=700 + i)
        W = wl.make_weights(N, K, wl.LLAMA, seed=800 + i)
        _, _, _, Y, acc = run_layer(X, W, G, a_in_tmem=bool(i % 2))
        r = oracle.linear(X.numpy(), W.numpy(), G)
        assert np.array_equal(acc.cpu().numpy(), r["acc"]), (M, K, N, G)


def test_empty_and_invalid_on_device():
    X = torch.zeros(0, 512, dtype=torch.float16, device="cuda")
    X8, s_x = q.qoq_quant_act_per_token(X)
    assert X8.shape == (0, 512)
    W = wl.make_weights(256, 512, wl.LLAMA, seed=7).cuda()
    p = q.qoq_pack_weights(W, 128)
    Y = q.qoq_w4a8_gemm(X8, s_x, p)
    assert Y.shape == (0, 256)
    with pytest.raises(q.QoQError):
        q.qoq_pack_weights(W, 64)
    small = torch.zeros(16, dtype=torch.uint8, device="cuda")
    X8b, s_xb = q.qoq_quant_act_per_token(wl.make_activations(4, 512, wl.LLAMA, 1).cuda())
    with pytest.raises(q.QoQError):
        q.qoq_w4a8_gemm(X8b, s_xb, p, workspace=small)


def test_output_and_accumulator_extremes():
    """Largest K with all-extreme inputs: |acc| reaches K*127*120 without
    overflow, both signs."""
    K = 24576
    X = torch.ones(2, K, dtype=torch.float16)
    X[1] = -1
    W = torch.ones(256, K)
    W[1::2] = -1
    _, _, _, Y, acc = run_layer(X, W, 128)
    r = oracle.linear(X.numpy(), W.numpy(), 128)
    assert np.array_equal(acc.cpu().numpy(), r["acc"])
    assert abs(int(r["acc"][0, 0])) == K * 127 * 120
    assert_half_within_1ulp(_u16(Y), r["Y"])
