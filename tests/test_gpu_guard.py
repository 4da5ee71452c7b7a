"""Guard bands around every buffer the kernels write: each output sits
between 4 KB of poisoned bytes, and after every launch those bytes must be
untouched.  The shapes reach every token-tile width (16 to 256, single CTAs
and CTA pairs), ragged M and both K-block widths, under both tile rules and
both forms of the layer call.  The outputs themselves are also compared with
the plain calls on ordinary buffers."""
import pytest
import torch

import w4a8_integer_gemm_b200 as q
from w4a8_integer_gemm_b200 import workloads as wl

pytestmark = pytest.mark.gpu

PAD = 4096
POISON = 0xA5


class Guarded:
    """A device buffer with PAD poisoned bytes on each side of `nbytes`."""

    def __init__(self, nbytes, fill=None):
        self.nbytes = nbytes
        self.raw = torch.full((PAD + nbytes + PAD,), POISON, dtype=torch.uint8, device="cuda")
        if fill is not None:
            self.raw[PAD:PAD + nbytes].fill_(fill)

    def view(self, dtype, shape):
        t = self.raw[PAD:PAD + self.nbytes].view(dtype)
        return t.view(*shape)

    def intact(self):
        return bool((self.raw[:PAD] == POISON).all()) and bool((self.raw[PAD + self.nbytes:] == POISON).all())


SHAPES = [
    # M, K, N, G
    (1, 512, 512, 128),      # 16-token tile, 256-wide K blocks
    (17, 1024, 384, 128),    # 32-token tile
    (33, 640, 256, 640),     # 64-token tile, 128-wide K blocks, per-channel tables
    (100, 512, 256, 128),    # 128-token tile (narrowed to 64 by default)
    (200, 768, 512, 128),    # 256-token tiles on CTA pairs (rule off), ragged M
    (300, 1024, 640, 128),   # 256-token tiles on single CTAs (N not a multiple of 256)
    (513, 512, 256, 512),    # three 256-token m-tiles on pairs
]


def _packed(W, G):
    N, K = W.shape
    nb = q.qoq_packed_weight_bytes(N, K, G)
    ng = K // G
    gw, gc = Guarded(nb), Guarded(2 * N)
    gg, gz = Guarded(N * ng), Guarded(N * ng)
    p = q.PackedWeights(gw.view(torch.uint8, (nb,)), gc.view(torch.int16, (N,)),
                        gg.view(torch.uint8, (N // 128, ng, 128)), gz.view(torch.uint8, (N // 128, ng, 128)),
                        N, K, G)
    q.qoq_pack_weights(W, G, out=p)
    return p, [gw, gc, gg, gz]


@pytest.mark.parametrize("M,K,N,G", SHAPES, ids=[f"M{m}_K{k}_N{n}_G{g}" for m, k, n, g in SHAPES])
def test_no_write_outside_any_buffer(M, K, N, G):
    q.qoq_set_gemm_a_in_tmem(True)
    dev = torch.device("cuda")
    X = wl.make_activations(M, K, wl.LLAMA, seed=7100 + M).to(dev)
    W = wl.make_weights(N, K, wl.LLAMA, seed=7200 + N).to(dev)
    ref_p = q.qoq_pack_weights(W, G)
    ref_X8, ref_sx = q.qoq_quant_act_per_token(X)
    ref_acc = torch.empty(M, N, dtype=torch.int32, device=dev)
    ref_Y = q.qoq_w4a8_gemm(ref_X8, ref_sx, ref_p, acc_dbg=ref_acc)
    torch.cuda.synchronize()

    p, guards = _packed(W, G)
    torch.cuda.synchronize()
    assert all(g.intact() for g in guards), "packer wrote outside its outputs"
    assert torch.equal(p.Wp, ref_p.Wp) and torch.equal(p.s_c, ref_p.s_c)
    assert torch.equal(p.s_g, ref_p.s_g) and torch.equal(p.zs, ref_p.zs)

    gx8, gsx = Guarded(M * K), Guarded(2 * M)
    X8, sx = gx8.view(torch.int8, (M, K)), gsx.view(torch.int16, (M,))
    q.qoq_quant_act_per_token(X, X8, sx)
    torch.cuda.synchronize()
    assert gx8.intact() and gsx.intact(), "quantizer wrote outside X8 / s_x"
    assert torch.equal(X8, ref_X8) and torch.equal(sx, ref_sx[:M])

    try:
        for narrow in (True, False):
            q.qoq_set_gemm_narrow_tiles(narrow)
            wsb = q.qoq_gemm_workspace_bytes(M, N, K, G)
            gws = Guarded(wsb, fill=0)
            gy, gacc = Guarded(2 * M * N), Guarded(4 * M * N)
            Y, acc = gy.view(torch.float16, (M, N)), gacc.view(torch.int32, (M, N))
            for run in range(2):
                q.qoq_w4a8_gemm(X8, sx, p, Y=Y, acc_dbg=acc, workspace=gws.view(torch.uint8, (wsb,)))
                torch.cuda.synchronize()
                assert q.qoq_device_error() == q.QOQ_OK
                assert gy.intact() and gacc.intact() and gws.intact(), f"GEMM wrote outside (narrow={narrow})"
                assert torch.equal(acc, ref_acc) and torch.equal(Y.view(torch.int16), ref_Y.view(torch.int16))
            for one_launch in (False, True):
                q.qoq_set_linear_in_kernel_quant(one_launch)
                gx8b, gsxb, gyb = Guarded(M * K), Guarded(2 * M), Guarded(2 * M * N)
                X8b, sxb = gx8b.view(torch.int8, (M, K)), gsxb.view(torch.int16, (M,))
                Yb = gyb.view(torch.float16, (M, N))
                q.qoq_w4a8_linear(X, p, X8=X8b, s_x=sxb, Y=Yb, workspace=gws.view(torch.uint8, (wsb,)))
                torch.cuda.synchronize()
                assert q.qoq_device_error() == q.QOQ_OK
                assert gx8b.intact() and gsxb.intact() and gyb.intact() and gws.intact(), \
                    f"layer call wrote outside (narrow={narrow}, one launch={one_launch})"
                assert torch.equal(Yb.view(torch.int16), ref_Y.view(torch.int16))
                assert torch.equal(X8b, ref_X8) and torch.equal(sxb, ref_sx[:M])
            # the workspace is left reusable: counters back at zero
            assert int(gws.view(torch.uint8, (wsb,))[:8192].view(torch.int32).abs().sum()) == 0
    finally:
        q.qoq_set_gemm_narrow_tiles(True)
        q.qoq_set_linear_in_kernel_quant(False)
