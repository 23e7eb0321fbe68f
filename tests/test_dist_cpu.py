"""The multi-rank host logic of bench.py on CPU: two gloo ranks (one process
each, as torchrun starts them) take the maximum of their timed regions, meet
at the barriers, and report the whole-job throughput of independent per-rank
token batches (weak scaling, no collective on the data path)."""
from __future__ import annotations

import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, out):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    w, r, local = bench.dist_env()
    assert (w, r, local) == (world, rank, rank)
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        bench.barrier(world)
        ms_local = 10.0 + 5.0 * rank             # rank 1 is the slow one
        ms = bench.max_over_ranks(ms_local, world)
        bench.barrier(world)
        value = bench.job_throughput(world, 8192, 100, ms)
        out.put((rank, ms, value))
    finally:
        dist.destroy_process_group()


def test_two_rank_max_over_ranks_and_weak_scaling_value():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    codes = [p.exitcode for p in procs]
    for p in procs:
        if p.is_alive():
            p.kill()
    assert codes == [0, 0], codes
    got = sorted(q.get(timeout=5) for _ in range(world))
    for rank, ms, value in got:
        assert ms == 15.0                         # every rank sees the slowest rank's time
        assert value == pytest.approx(2 * 8192 * 100 / 0.015)


def test_single_rank_helpers_are_identities():
    import bench
    assert bench.max_over_ranks(3.25, 1) == 3.25
    bench.barrier(1)
    assert bench.job_throughput(1, 8192, 2000, 194.2) == pytest.approx(8192 * 2000 / 0.1942)
