"""The multi-rank plumbing of bench.py on CPU with gloo (world size 2): each
rank scores its own units (own seed, weak scaling), the step time is the max
over ranks, and the job value counts every rank's units."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        local_ms = 100.0 + 25.0 * rank            # rank 1 is the slowest
        mx = bench.max_over_ranks(local_ms, world, "cpu")
        seeds = [None] * world
        dist.all_gather_object(seeds, bench.rank_seed(7, rank))
        out[rank] = (mx, seeds)
    finally:
        dist.destroy_process_group()


def test_two_rank_gloo_plumbing():
    world = 2
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, port, out), nprocs=world, start_method="spawn", join=True)
    for r in range(world):
        mx, seeds = out[r]
        assert mx == 125.0                          # max over ranks, the same on every rank
        assert len(set(seeds)) == world            # every rank its own units
    import bench
    # value = all ranks' units over the slowest rank's time
    assert bench.whole_job_value(2, 1000, 10, 125.0) == pytest.approx(2 * 1000 * 10 / 0.125)


def test_single_rank_is_identity():
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.rank_seed(5, 0) == 5
