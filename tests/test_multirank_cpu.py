"""The bench's multi-rank host logic on two CPU ranks (gloo): every rank takes the
same collective steps and the reported time is the maximum over ranks."""

import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, results):
    import datetime

    import torch
    import torch.distributed as dist

    import bench

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    w, r, local = bench.dist_env()
    assert (w, r, local) == (world, rank, rank)
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    try:
        cpu = torch.device("cpu")
        bench.barrier(cpu)
        per_rank_ms = [12.5, 30.25][rank]
        got = bench.max_over_ranks(per_rank_ms, cpu)
        bench.barrier(cpu)
        results[rank] = got
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_max_over_two_gloo_ranks():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        results = m.dict()
        procs = [ctx.Process(target=_worker, args=(r, world, port, results)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(100)
        assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
        assert dict(results) == {0: 30.25, 1: 30.25}


def test_single_rank_is_identity():
    import torch

    import bench

    assert bench.max_over_ranks(7.0, torch.device("cpu")) == 7.0
