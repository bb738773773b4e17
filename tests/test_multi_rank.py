"""Multi-rank host logic of the benchmark on CPU (gloo, world size 2): each
rank runs its own layer, the job time is the slowest rank's, and throughput is
every rank's tokens over that time.  The operator itself has no collective."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from clustered_multipole_approximation_b200.inputs import WORKLOADS


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = [120.0, 150.0][rank]
        m = bench.max_over_ranks(local_ms, world)
        w = WORKLOADS["acausal-bf16-h8-n8k"]
        out[rank] = (m, bench.rank_data_seed(w, rank),
                     bench.whole_job_throughput(w.B * w.N, world, 10, m))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_ranks_take_the_slowest_time():
    world = 2
    mgr = mp.Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, start_method="spawn")
    assert out[0][0] == out[1][0] == 150.0
    assert out[0][1] != out[1][1]          # independent layers per rank
    assert out[0][2] == pytest.approx(8192 * 2 * 10 / 0.150)


def test_single_rank_is_identity():
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.whole_job_throughput(100, 1, 4, 2000.0) == pytest.approx(200.0)
