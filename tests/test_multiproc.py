"""The replica path of bench.py on CPU: two gloo ranks, max-over-ranks timing, whole-job throughput."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    r, lr, w = bench.dist_env()
    seconds = 0.010 * (rank + 1)            # rank 1 is the slow one
    m = bench.reduce_max(seconds, w)
    q.put((r, lr, w, m, bench.aggregate(8 * 20, m, w)))
    dist.barrier()
    dist.destroy_process_group()


def test_two_replicas_max_over_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[0] for r in res] == [0, 1] and all(r[2] == 2 for r in res)
    for r in res:
        assert r[3] == pytest.approx(0.020)               # both ranks see the slowest time
        assert r[4] == pytest.approx(8 * 20 * 2 / 0.020)  # tokens of both replicas / that time


def test_single_rank_identity():
    import bench
    assert bench.reduce_max(1.25, 1) == 1.25
    assert bench.aggregate(100, 2.0, 1) == 50.0
