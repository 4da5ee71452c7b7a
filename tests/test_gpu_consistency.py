"""Every output of the GEMM, checked at full size, over repeated runs.

The sampled full-size parity tests compare a few thousand outputs per shape
with the oracle; this test covers all of them through a property that holds
at any size: the INT32 accumulators equal X8 . W8hat^T exactly, where X8
comes from the activation quantizer and W8hat from qoq_dequant_weights_i8
(both checked bit for bit against the oracle elsewhere), multiplied by
torch's INT8 matmul (cuBLASLt, INT32 accumulation).  The FP16 outputs must
then equal fp16(((float)acc * s_x) * s_c), computed elementwise by torch in
FP32.  Each shape runs several times, eagerly and from a CUDA graph, and
every run must match: a missed handoff between CTAs (a split tile whose
partial is read before it is visible) shows up here as whole-channel errors.
"""
import pytest
import torch

import w4a8_integer_gemm_b200 as q
from w4a8_integer_gemm_b200 import workloads as wl

pytestmark = pytest.mark.gpu

SHAPES = [
    # M, K, N, G
    (1, 4096, 14336, 128),
    (8, 4096, 14336, 4096),
    (32, 4096, 14336, 128),
    (64, 4096, 14336, 4096),
    (64, 4096, 14336, 128),
    (100, 4096, 6144, 128),
    (256, 4096, 4096, 128),
    (1024, 4096, 4096, 128),
]


def _ref_acc(X8, W8):
    M = X8.shape[0]
    Mp = max(32, (M + 7) // 8 * 8)
    A = torch.zeros(Mp, X8.shape[1], dtype=torch.int8, device=X8.device)
    A[:M] = X8
    return torch._int_mm(A, W8.t())[:M]


def _ref_y(acc, s_x, s_c):
    sx = s_x[: acc.shape[0]].view(torch.float16).float()
    sc = s_c.view(torch.float16).float()
    return ((acc.float() * sx[:, None]) * sc[None, :]).half()


@pytest.mark.parametrize("M,K,N,G", SHAPES, ids=[f"M{m}_K{k}_N{n}_G{g}" for m, k, n, g in SHAPES])
def test_all_outputs_repeated(M, K, N, G):
    q.qoq_set_gemm_a_in_tmem(True)
    dev = torch.device("cuda")
    X = wl.make_activations(M, K, wl.LLAMA, seed=5100 + M).to(dev)
    W = wl.make_weights(N, K, wl.LLAMA, seed=5200 + M + G)
    packed = q.qoq_pack_weights(W.to(dev), G)
    del W
    X8, s_x = q.qoq_quant_act_per_token(X)
    W8 = q.qoq_dequant_weights_i8(packed)
    ref = _ref_acc(X8, W8)
    yref = _ref_y(ref, s_x, packed.s_c)
    del W8

    acc = torch.empty(M, N, dtype=torch.int32, device=dev)
    Y = torch.empty(M, N, dtype=torch.float16, device=dev)
    ws = torch.zeros(q.qoq_gemm_workspace_bytes(M, N, K, G), dtype=torch.uint8, device=dev)
    for run in range(4):
        acc.fill_(-7)
        Y.fill_(0)
        q.qoq_w4a8_gemm(X8, s_x, packed, Y=Y, acc_dbg=acc, workspace=ws)
        torch.cuda.synchronize()
        assert q.qoq_device_error() == q.QOQ_OK
        bad = (acc != ref)
        if bad.any():
            rows, cols = torch.nonzero(bad, as_tuple=True)
            pytest.fail(f"run {run}: {int(bad.sum())} INT32 mismatches in {rows.unique().numel()} tokens x "
                        f"{cols.unique().numel()} channels, first channels {cols.unique()[:8].tolist()}")
        assert torch.equal(Y.view(torch.int16), yref.view(torch.int16)), f"run {run}: FP16 outputs differ"

    # the same launches replayed from a CUDA graph (no acc_dbg: the serving call)
    main = torch.cuda.current_stream()
    cap = torch.cuda.Stream()
    cap.wait_stream(main)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=cap):
        q.qoq_quant_act_per_token(X, X8, s_x, stream=cap)
        q.qoq_w4a8_gemm(X8, s_x, packed, Y=Y, workspace=ws, stream=cap)
    main.wait_stream(cap)
    for run in range(4):
        Y.fill_(0)
        g.replay()
        torch.cuda.synchronize()
        assert q.qoq_device_error() == q.QOQ_OK
        assert torch.equal(Y.view(torch.int16), yref.view(torch.int16)), f"graph replay {run}: outputs differ"
    del g
    assert int(ws[:8192].view(torch.int32).abs().sum()) == 0


PAIR_SHAPES = [(200, 1024, 512, 128), (256, 4096, 4096, 128), (513, 512, 256, 512), (1024, 4096, 4096, 128), (4096, 2048, 1024, 128)]


@pytest.mark.parametrize("M,K,N,G", PAIR_SHAPES, ids=[f"M{m}_K{k}_N{n}_G{g}" for m, k, n, g in PAIR_SHAPES])
def test_cta_pairs_match_single(M, K, N, G):
    """256-token tiles on CTA pairs (2-SM MMA, A in TMEM or in shared
    memory) give the same bits as on single CTAs, and as the narrower tiles
    the default rule picks for few tiles; all equal the exact product."""
    dev = torch.device("cuda")
    X = wl.make_activations(M, K, wl.LLAMA, seed=5300 + M)
    W = wl.make_weights(N, K, wl.LLAMA, seed=5400 + M)
    packed = q.qoq_pack_weights(W.to(dev), G)
    X8, s_x = q.qoq_quant_act_per_token(X.to(dev))
    ref = _ref_acc(X8, q.qoq_dequant_weights_i8(packed))
    out = {}
    try:
        for a_tmem in (True, False):
            q.qoq_set_gemm_a_in_tmem(a_tmem)
            for narrow, pairs in ((False, False), (False, True), (True, True)):
                q.qoq_set_gemm_narrow_tiles(narrow)
                q.qoq_set_gemm_cta_pairs(pairs)
                for run in range(3):
                    acc = torch.full((M, N), -7, dtype=torch.int32, device=dev)
                    Y = q.qoq_w4a8_gemm(X8, s_x, packed, acc_dbg=acc)
                    torch.cuda.synchronize()
                    assert q.qoq_device_error() == q.QOQ_OK
                    assert torch.equal(acc, ref), f"a_tmem={a_tmem} narrow={narrow} pairs={pairs} run {run}"
                out[(a_tmem, narrow, pairs)] = Y
    finally:
        q.qoq_set_gemm_cta_pairs(True)
        q.qoq_set_gemm_narrow_tiles(True)
        q.qoq_set_gemm_a_in_tmem(True)
    for k in out:
        assert torch.equal(out[k].view(torch.int16), out[(True, False, False)].view(torch.int16)), k
