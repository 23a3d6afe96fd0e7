"""The multi-GPU bench path is replicas only: each rank runs its own batch,
no collective touches the data, and the reported time is the max over ranks.
The timing reduction is checked here with two gloo ranks on the CPU."""
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    bench.barrier(world)
    t = bench.max_over_ranks(world, 1.5 + rank)          # rank r measured 1.5 + r ms
    results[rank] = t
    bench.barrier(world)
    dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_max_over_ranks_two_gloo_ranks():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    results = ctx.Manager().dict()
    procs = [ctx.Process(target=_worker, args=(r, world, port, results)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(100)
        assert p.exitcode == 0
    assert dict(results) == {0: 2.5, 1: 2.5}


def test_single_rank_is_identity():
    import bench
    assert bench.max_over_ranks(1, 3.25) == 3.25
