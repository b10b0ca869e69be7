"""The N > 1 host logic of bench.py on CPU: two gloo ranks (one process each,
as torchrun would start them) shard the inputs by rank, agree on the slowest
rank's time and report the whole-job throughput."""
import os
import socket

import pytest
import torch
import torch.distributed as td
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    import datetime

    import bench
    td.init_process_group("gloo", rank=rank, world_size=world,
                          timeout=datetime.timedelta(seconds=60))
    try:
        # every rank sees the max of the per-rank device times
        got = bench.rank_max(td, [10.0 + rank, 5.0 - rank], "cpu")
        # inputs are sharded: each rank draws its own seeded batch
        x, q = bench.make_inputs(bench.CONFIGS["tiny"], "cpu", seed_offset=rank, max_rows=64)
        xs = [torch.empty_like(x) for _ in range(world)]
        td.all_gather(xs, x)
        out[rank] = (got, bool(torch.equal(xs[0], xs[1])))
    finally:
        td.destroy_process_group()


def test_two_gloo_ranks():
    world, port = 2, _free_port()
    out = mp.Manager().dict()
    mp.spawn(_rank_main, args=(world, port, out), nprocs=world, join=True)
    for rank in range(world):
        got, same = out[rank]
        assert got == [11.0, 5.0]
        assert not same  # the ranks' batches differ


def test_job_throughput_counts_every_rank():
    import bench
    # 2 ranks x 1000 units x 10 steps in 20 ms (slowest rank) -> 1 Mvec/s
    assert bench.job_throughput(1000, 2, 10, 20.0) == pytest.approx(1.0)
    assert bench.rank_max(None, [3.0, 4.0], "cpu") == [3.0, 4.0]
