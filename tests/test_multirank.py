"""The multi-rank plumbing of bench.py on CPU: two gloo ranks (no GPU).

Each rank runs an independent batch (the path shards by sequence with no
exchange), so the only cross-rank steps are the barriers around the timed
region and the reductions of the report: time = max over ranks, bytes and
sequences = sum over ranks.
"""
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        bench.barrier(world)
        t = bench.max_over_ranks(1.5 + rank, world)          # rank 1 is the slow one
        b = bench.sum_over_ranks(1000.0 * (rank + 1), world)  # bytes of both ranks
        out.put((rank, t, b))
        bench.barrier(world)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_reduce_time_max_and_work_sum():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    for rank, t, b in res:
        assert t == 2.5
        assert b == 3000.0
