"""The row-parallel (K-split) layer's host logic on the CPU.

* the K slices cover [0, K) in whole 128-wide blocks;
* slicing a packed weight gives exactly the packed layout of the sliced
  codes and tables (the layout reference of include/qoq.h, built with numpy);
* with two gloo ranks, summing the ranks' INT32 partial sums through the
  module's all-reduce and scaling once reproduces the oracle's whole layer
  bit for bit (the partials are the oracle's own products on each slice).
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle
from layout_ref import pack_reference, tables_reference
from w4a8_integer_gemm_b200 import PackedWeights, tp
from w4a8_integer_gemm_b200 import workloads as wl


@pytest.mark.parametrize("K,world", [(128, 1), (4096, 2), (4096, 3), (14336, 8), (24576, 5)])
def test_k_slices_partition(K, world):
    sl = tp.k_slices(K, world)
    assert len(sl) == world and sl[0][0] == 0 and sl[-1][1] == K
    for (a, b), (c, d) in zip(sl, sl[1:]):
        assert b == c
    sizes = [b - a for a, b in sl]
    assert all(s % 128 == 0 and s > 0 for s in sizes)
    assert max(sizes) - min(sizes) <= 128


def test_k_slices_rejects():
    with pytest.raises(ValueError):
        tp.k_slices(256, 3)
    with pytest.raises(ValueError):
        tp.k_slices(300, 1)


def _packed_cpu(N, K, G, seed):
    W = wl.make_weights(N, K, wl.LLAMA, seed=seed).numpy()
    r = oracle.quantize_weights(W, G)
    Wp = pack_reference(r["q"], G, r["s_g"], r["zs"])
    p = PackedWeights(torch.from_numpy(Wp.copy()), torch.from_numpy(r["s_c"].view(np.int16).copy()),
                      torch.from_numpy(tables_reference(r["s_g"])), torch.from_numpy(tables_reference(r["zs"])),
                      N, K, G)
    return r, p


@pytest.mark.parametrize("G", [128, "K"])
def test_shard_packed_matches_layout_of_sliced_codes(G):
    N, K = 256, 1024
    G = K if G == "K" else G
    r, p = _packed_cpu(N, K, G, seed=3)
    for (k0, k1) in tp.k_slices(K, 3):
        sh = tp.shard_packed(p, k0, k1)
        assert sh.K == k1 - k0 and sh.N == N
        if G == 128:
            want = pack_reference(np.ascontiguousarray(r["q"][:, k0:k1]), 128,
                                  np.ascontiguousarray(r["s_g"][:, k0 // 128:k1 // 128]),
                                  np.ascontiguousarray(r["zs"][:, k0 // 128:k1 // 128]))
            assert sh.group_size == 128
            assert np.array_equal(sh.s_g.numpy(), tables_reference(r["s_g"][:, k0 // 128:k1 // 128]))
        else:
            want = pack_reference(np.ascontiguousarray(r["q"][:, k0:k1]), k1 - k0)
            assert sh.group_size == k1 - k0
            assert np.array_equal(sh.s_g.numpy(), tables_reference(r["s_g"]))
        assert np.array_equal(sh.Wp.numpy(), want)


def test_per_channel_slice_of_one_block_rejected():
    r, p = _packed_cpu(128, 512, 512, seed=4)
    with pytest.raises(ValueError):
        tp.shard_packed(p, 0, 128)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import datetime
    import torch.distributed as dist
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    try:
        M, N, K, G = 9, 256, 1024, 128
        X = wl.make_activations(M, K, wl.LLAMA, seed=11)
        W = wl.make_weights(N, K, wl.LLAMA, seed=12)
        full = oracle.linear(X.numpy(), W.numpy(), G)
        k0, k1 = tp.k_slices(K, world)[rank]
        # this rank's partial sums: the oracle's products on its slice of the
        # (replicated) INT8 activations and the dequantized weights
        part = oracle.gemm_i32(np.ascontiguousarray(full["X8"][:, k0:k1]),
                               np.ascontiguousarray(full["W8hat"][:, k0:k1]))
        acc = torch.from_numpy(part.copy())
        tp.allreduce_partials(acc)
        Y = oracle.epilogue(acc.numpy(), full["s_x"], full["s_c"])
        out.put((rank, bool(np.array_equal(acc.numpy(), full["acc"])), bool(np.array_equal(Y, full["Y"])),
                 bool(np.array_equal(part, full["acc"]))))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(180)
@pytest.mark.parametrize("world", [2, 3])
def test_ranks_sum_to_the_single_gpu_layer(world):
    ctx = mp.get_context("spawn")
    qu = ctx.Queue()
    port = _free_port()
    ps = [ctx.Process(target=_worker, args=(r, world, port, qu)) for r in range(world)]
    for p in ps:
        p.start()
    res = sorted(qu.get(timeout=150) for _ in range(world))
    for p in ps:
        p.join(timeout=30)
        assert p.exitcode == 0
    for rank, acc_ok, y_ok, part_is_full in res:
        assert acc_ok and y_ok
        assert not part_is_full          # each rank alone has only a partial sum
