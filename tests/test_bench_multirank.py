"""The multi-rank host logic of bench.py on CPU: two gloo ranks, timings reduced to the
maximum over ranks, the whole-job rate counts every rank's units."""

import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    mine = [10.0 + 5.0 * rank, 3.0 - rank]          # rank 1 slower in the first, faster in the second
    got = bench.max_over_ranks(mine, torch.device("cpu"), True)
    out[rank] = got
    dist.barrier()
    dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_rank, args=(2, port, out), nprocs=2, start_method="spawn", join=True)
    assert out[0] == [15.0, 3.0] and out[1] == [15.0, 3.0]


def test_whole_job_rate_and_single_process():
    import bench
    assert bench.whole_job_rate(4, 32, 2.0) == pytest.approx(4 * 32 / 2e-3)
    assert bench.max_over_ranks([1.5, 2.5], torch.device("cpu"), False) == [1.5, 2.5]
