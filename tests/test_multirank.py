"""The bench's multi-rank host logic on CPU: two gloo ranks.

Attention heads are independent, so ranks share no data-path collective; the only
cross-rank steps are the timing barrier and the max over ranks of the measured times.
"""

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    # rank r measured (r + 1) ms for the step and 10 - r ms for the forward
    mx = bench.max_over_ranks([1.0 + rank, 10.0 - rank])
    dist.barrier()
    out[rank] = mx
    dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    world = 2
    port = _free_port()
    manager = mp.get_context("spawn").Manager()
    out = manager.dict()
    mp.start_processes(_worker, args=(world, port, out), nprocs=world, join=True, start_method="spawn")
    assert out[0] == [2.0, 10.0] and out[1] == [2.0, 10.0]


def test_single_process_is_identity_and_throughput_counts_all_ranks():
    import bench
    assert bench.max_over_ranks([3.0, 4.5]) == [3.0, 4.5]
    one = bench.job_throughput(1, 1e12, 1000.0)
    assert one == pytest.approx(1.0)
    assert bench.job_throughput(8, 1e12, 1000.0) == pytest.approx(8 * one)
