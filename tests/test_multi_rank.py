"""The N > 1 path of bench.py on CPU: two gloo ranks.

The layer needs no exchange between GPUs: each rank runs the whole workload
on its own device (replicas, weak scaling). What the multi-rank path adds is
host logic, tested here without a GPU:
- the time is the maximum over ranks;
- the value is the bytes of all ranks over that time;
- every rank takes the same collective steps.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    import torch.distributed as dist

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import bench

    try:
        bench.init_dist(world, "gloo")
        r, lr, w = bench.dist_env()
        per_rank_bytes = 1000.0 * (rank + 1)
        per_rank_seconds = 0.5 + rank  # rank 1 is the slowest
        total, tmax, value = bench.aggregate(per_rank_bytes, per_rank_seconds)
        bench.barrier()
        mx = bench.reduce_over_ranks(float(rank), "max")
        sm = bench.reduce_over_ranks(1.0, "sum")
        q.put((rank, r, w, total, tmax, value, mx, sm))
    finally:
        if dist.is_initialized():
            dist.destroy_process_group()


def test_two_rank_aggregation_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, r, w, total, tmax, value, mx, sm in out:
        assert r == rank and w == 2
        assert total == 3000.0          # bytes of both ranks
        assert tmax == 1.5              # the slowest rank's time
        assert value == pytest.approx(2000.0)
        assert mx == 1.0 and sm == 2.0


def test_single_rank_is_identity():
    import bench

    total, tmax, value = bench.aggregate(10.0, 2.0)
    assert (total, tmax, value) == (10.0, 2.0, 5.0)
