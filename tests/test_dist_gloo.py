"""The benchmark's multi-rank host logic on CPU: two gloo ranks on
127.0.0.1 (replicas, no data-path collective).  Each rank reports a
different step time; the job's time must be the slowest rank's and the
value all ranks' work over it."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import datetime
    import torch.distributed as dist
    import bench
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    try:
        ms_mine = 2.0 + 3.0 * rank          # rank 1 is the slow one
        ms, value = bench.aggregate(1e12, ms_mine, world, dist)
        bench.barrier(dist)
        q.put((rank, ms, value))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_two_rank_aggregate_takes_max():
    world = 2
    ctx = mp.get_context("spawn")
    qu = ctx.Queue()
    port = _free_port()
    ps = [ctx.Process(target=_worker, args=(r, world, port, qu)) for r in range(world)]
    for p in ps:
        p.start()
    res = sorted(qu.get(timeout=90) for _ in range(world))
    for p in ps:
        p.join(timeout=30)
        assert p.exitcode == 0
    for rank, ms, value in res:
        assert ms == pytest.approx(5.0)                       # slowest rank
        assert value == pytest.approx(2 * 1e12 / 5e-3 / 1e12)  # 400 TOPS
