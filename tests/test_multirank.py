"""The benchmark's multi-rank path on CPU: two gloo ranks, as `bench.py --gpus 2` runs two
NCCL ranks. Each rank processes its own replica of the independent (sequence, KV head)
units, so there is no data-path collective; the only exchange is the element-wise maximum of
the per-rank timings, and the job's throughput counts every rank's units over the slowest
rank's time."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, result_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        mine = [10.0 + rank, 3.0 - rank, 5.0 * (rank + 1), 7.0]
        got = bench.max_over_ranks(mine, torch.device("cpu"))
        with open(os.path.join(result_dir, f"r{rank}.txt"), "w") as f:
            f.write(",".join(repr(x) for x in got))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_timings_take_the_slowest_rank(tmp_path):
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, start_method="spawn")
    for r in range(world):
        vals = [float(x) for x in (tmp_path / f"r{r}.txt").read_text().split(",")]
        assert vals == [11.0, 3.0, 10.0, 7.0]


def test_single_rank_timings_pass_through():
    assert bench.max_over_ranks([1.5, 2.5], torch.device("cpu")) == [1.5, 2.5]


def test_job_throughput_counts_every_rank():
    one = bench.job_throughput(1, 36, 1, 131072, 5.0)
    two = bench.job_throughput(2, 36, 1, 131072, 5.0)
    assert two == pytest.approx(2 * one)
    assert one == pytest.approx(36 * 131072 / 5e-3)
