"""Host-side logic of bench.py's replica mode, on 2 gloo ranks (CPU only)."""

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
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench

    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = [4.0, 10.0][rank]
        value, ms_max = bench.aggregate_throughput(1e9, ms, world)
        bench.barrier(world)
        q.put((rank, value, ms_max, bench.max_over_ranks(float(rank), world)))
    finally:
        dist.destroy_process_group()


def test_replicas_take_max_over_ranks_and_sum_units():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, value, ms_max, mx in res:
        assert ms_max == 10.0                      # the slowest rank's time
        assert value == pytest.approx(2e9 / 10e-3)  # all ranks' units over that time
        assert mx == 1.0


def test_single_rank_is_identity():
    import bench

    value, ms = bench.aggregate_throughput(5e8, 2.0, 1)
    assert ms == 2.0 and value == pytest.approx(5e8 / 2e-3)
