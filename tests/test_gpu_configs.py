"""Parity at the workloads' full sizes, in the launch configuration the
benchmark times (cached workspace, A operand in TMEM, current stream).

Every shape of every workload runs the whole GPU path once; the oracle then
recomputes a sample of outputs one by one (48 tokens x 64 channels, chosen
by a seeded generator and always including the first and last token and
channel), which must match the INT32 accumulators bit for bit and the FP16
outputs to 1 ulp.  The packed weights of each distinct (N, K, group) are
also compared in full against the oracle's codes.
"""
import numpy as np
import pytest
import torch

import oracle
import w4a8_integer_gemm_b200 as q
from w4a8_integer_gemm_b200 import workloads as wl
from layout_ref import pack_reference, tables_reference

pytestmark = pytest.mark.gpu

CASES = [(name, i) for name, w in wl.WORKLOADS.items() for i in range(len(w.shapes))]
_packed_checked = set()


def _sample(n, k, rng):
    idx = rng.choice(n, size=min(k, n), replace=False)
    return np.unique(np.concatenate([idx, [0, n - 1]]))


@pytest.mark.parametrize("name,i", CASES, ids=[f"{n}-{wl.WORKLOADS[n].shapes[i].name}" for n, i in CASES])
def test_full_size_sampled(name, i):
    q.qoq_set_gemm_a_in_tmem(True)
    w = wl.WORKLOADS[name]
    s = w.shapes[i]
    X, W = wl.make_case(w, i)
    Wd = W.cuda()
    packed = q.qoq_pack_weights(Wd, s.G)
    X8, s_x = q.qoq_quant_act_per_token(X.cuda())
    acc = torch.empty(s.M, s.N, dtype=torch.int32, device="cuda")
    Y = q.qoq_w4a8_gemm(X8, s_x, packed, acc_dbg=acc)
    torch.cuda.synchronize()
    assert q.qoq_device_error() == q.QOQ_OK
    del Wd

    rng = np.random.default_rng(1000 * w.number + i)
    rows = _sample(s.M, 48, rng)
    cols = _sample(s.N, 64, rng)
    r = oracle.linear_sampled(X.numpy(), W.numpy(), s.G, rows, cols)
    got_acc = acc[torch.as_tensor(rows)][:, torch.as_tensor(cols)].cpu().numpy()
    assert np.array_equal(got_acc, r["acc"])
    got_y = Y[torch.as_tensor(rows)][:, torch.as_tensor(cols)].cpu().view(torch.int16).numpy().view(np.uint16)
    g = got_y.view(np.float16).astype(np.float64)
    ref = r["Y"].view(np.float16).astype(np.float64)
    ulp = np.spacing(np.abs(ref).astype(np.float16)).astype(np.float64)
    assert np.all(np.abs(g - ref) <= ulp)
    # the sampled tokens' INT8 activations and scales, bit for bit
    assert np.array_equal(X8[torch.as_tensor(rows)].cpu().numpy(), r["X8"])

    key = (s.N, s.K, s.G, w.number)
    if key not in _packed_checked:
        _packed_checked.add(key)
        full = oracle.quantize_weights(W.numpy(), s.G)
        assert np.array_equal(packed.s_c.cpu().view(torch.int16).numpy().view(np.uint16), full["s_c"])
        assert np.array_equal(packed.s_g.cpu().numpy(), tables_reference(full["s_g"]))
        assert np.array_equal(packed.zs.cpu().numpy(), tables_reference(full["zs"]))
        assert np.array_equal(packed.Wp.cpu().numpy(), pack_reference(full["q"], s.G, full["s_g"], full["zs"]))
