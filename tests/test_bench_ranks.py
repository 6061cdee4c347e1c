"""CPU: the host logic of the multi-process bench path (one process per GPU,
replicas) on two gloo ranks: the job's time is the slowest rank's, seen by
every rank, and the job's throughput counts every rank's units."""
import os
import socket
from datetime import timedelta

import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, times, out_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        import bench

        got = bench.max_over_ranks(times[rank], world, torch.device("cpu"))
        # a second collective in the same order on every rank (the bench's e2e timing)
        got2 = bench.max_over_ranks(times[world - 1 - rank] * 2.0, world, torch.device("cpu"))
        with open(os.path.join(out_dir, f"rank{rank}"), "w") as f:
            f.write(f"{got!r} {got2!r}")
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_on_two_gloo_ranks(tmp_path):
    times = [3.25, 5.5]
    mp.spawn(_worker, args=(2, _free_port(), times, str(tmp_path)), nprocs=2, join=True)
    for r in range(2):
        got, got2 = (float(x) for x in (tmp_path / f"rank{r}").read_text().split())
        assert got == 5.5
        assert got2 == 11.0


def test_job_throughput_counts_every_rank():
    import bench

    assert bench.job_throughput(1, 8.0e12, 8.0) == 1.0e15
    # four replicas, each 8e12 units in 8 ms: four times the single-rank rate
    assert bench.job_throughput(4, 8.0e12, 8.0) == 4.0e15
    assert bench.max_over_ranks(7.0, 1, torch.device("cpu")) == 7.0


def test_reference_arm_runs_on_rank_zero_only():
    """Under a multi-process launch the oracle's reference arm runs on rank 0
    alone; other ranks return at once without work (and print nothing)."""
    import argparse

    import bench

    args = argparse.Namespace(workload="dflash_long_full", steps=1, warmup=3)
    assert bench.run_reference(args, 1, 2) is None
