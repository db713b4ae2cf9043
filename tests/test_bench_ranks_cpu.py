"""The multi-rank plumbing of bench.py on CPU: two gloo ranks agree on the
slowest rank's time, the whole-job rate counts every rank's replica, and the
reference arm runs on rank 0 only."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import datetime
    import torch.distributed as dist
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        dist.barrier()
        ms = bench.max_over_ranks(10.0 * (rank + 1) + 0.25)     # rank r took 10 (r + 1) + 0.25 ms
        out[rank] = (ms, bench.job_rate(world, 5, ms))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_rate_two_gloo_ranks():
    world = 2
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True)
    for r in range(world):
        ms, rate = out[r]
        assert ms == pytest.approx(20.25)                       # the slowest rank's time, on every rank
        assert rate == pytest.approx(world * 5 / 0.02025)        # both replicas' steps over that time


def test_single_process_unchanged():
    import bench
    assert bench.max_over_ranks(12.5) == 12.5
    assert bench.job_rate(1, 4, 500.0) == pytest.approx(8.0)


def test_reference_arm_prints_on_rank0_only(capsys):
    import argparse
    import bench
    args = argparse.Namespace(workload=1, shapes=None, warmup=0, steps=1, gpus=2)
    bench.run_reference(args, rank=1, world=2)
    assert capsys.readouterr().out == ""
