"""Host logic of the multi-GPU benchmark on CPU: two gloo ranks (world size 2)
exercise the max-over-ranks reduction and the per-rank problem seeds that
bench.py uses when launched under torchrun (no GPU involved)."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import datetime

    import torch.distributed as dist

    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        r, w, lr = bench.dist_env()
        assert (r, w, lr) == (rank, world, rank)
        # rank-dependent timings: the maximum over ranks is reported everywhere
        got = bench.reduce_max([1.0 + rank, 10.0 - rank, 3.0], world)
        out[rank] = (got, bench.rank_seed(4, rank))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_rank_reduction_and_seeds():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    for r in range(world):
        got, seed = out[r]
        assert got == [2.0, 10.0, 3.0]
    # each rank draws an independent problem
    assert out[0][1] != out[1][1]


def test_single_rank_reduction_is_identity():
    import bench
    assert bench.reduce_max([1.5, 2.5], 1) == [1.5, 2.5]
