"""Multi-rank plumbing of the benchmark on CPU (gloo, world size 2): every rank prunes its
own layer and the job's throughput uses the slowest rank's device time."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    local_ms = [100.0, 250.0][rank]
    value, max_ms = bench.job_throughput(local_ms, world, 4096 * 4096, 10)
    out[rank] = (value, max_ms)
    dist.barrier()
    dist.destroy_process_group()


def test_job_throughput_takes_slowest_rank_and_sums_work():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, start_method="spawn")
    assert out[0] == out[1]
    value, max_ms = out[0]
    assert max_ms == 250.0
    assert value == pytest.approx(2 * 4096 * 4096 * 10 / 0.25)


def test_single_rank_throughput():
    import bench
    value, max_ms = bench.job_throughput(50.0, 1, 1000, 4)
    assert max_ms == 50.0 and value == pytest.approx(1000 * 4 / 0.05)
