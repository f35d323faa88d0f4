"""The benchmark's multi-rank logic on CPU with two gloo ranks: every rank
draws its own batch, timings are the maximum over ranks, the job throughput
counts the bytes of all ranks, and the reference arm runs on rank 0 only."""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    sys.path.insert(0, ROOT)
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # rank r's step time is 1 + r ms: the job runs at the slowest rank
        slowest = bench.max_over_ranks(1.0 + rank, dist, torch.device("cpu"))
        seeds = [None] * world
        dist.all_gather_object(seeds, bench.rank_seed(7, rank))
        out[rank] = (slowest, tuple(seeds))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_max_and_draw_distinct_batches():
    world = 2
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.start_processes(_rank_main, args=(world, _free_port(), out), nprocs=world,
                           start_method="spawn", join=True)
        res = dict(out)
    assert set(res) == {0, 1}
    for r in range(world):
        slowest, seeds = res[r]
        assert slowest == 2.0                 # both ranks see the slowest rank's time
        assert len(set(seeds)) == world       # independent batches per rank


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, None, None) == 3.5


def test_job_throughput_counts_every_rank():
    sys.path.insert(0, ROOT)
    import bench
    # 1 GB per rank in 2 ms on each of 4 ranks: 4 GB / 2 ms = 2000 GB/s
    assert bench.job_throughput(1e9, 4, 2.0) == pytest.approx(2000.0)
    assert bench.job_throughput(1e9, 1, 2.0) == pytest.approx(500.0)


def test_reference_arm_runs_on_rank_zero_only(capsys):
    sys.path.insert(0, ROOT)
    import bench
    bench.run_reference(None, rank=1)         # returns before touching args
    assert capsys.readouterr().out == ""
