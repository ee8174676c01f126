"""The multi-GPU host logic of bench.py on CPU: two ranks over gloo (127.0.0.1).

bench.py runs one process per GPU on independent sequences (replicas, no data-path
collective); the only cross-rank steps are the timing reductions.  These tests run those
steps with two gloo ranks and check the job-level numbers: the step time is the slowest
rank's, the end-to-end rate is the slowest rank's rate times the rank count, and each rank
draws its own inputs."""
import importlib.util
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    return m


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        b = _bench()
        ms = b.max_over_ranks(10.0 + 5.0 * rank, world, torch.device("cpu"))  # rank 1 is slower
        rate = b.job_rate(100.0 - 30.0 * rank, world, torch.device("cpu"))
        dist.barrier()
        out[rank] = (ms, rate, b.rank_seed(rank), b.rank_seed(rank, 3))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_reduce_like_the_job():
    world = 2
    out = mp.get_context("spawn").Manager().dict()
    mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, start_method="spawn", join=True)
    assert out[0][0] == out[1][0] == 15.0              # slowest rank's time
    assert out[0][1] == out[1][1] == 70.0 * world      # slowest rank's rate x ranks
    seeds = {out[0][2], out[1][2], out[0][3], out[1][3]}
    assert len(seeds) == 4                              # every rank and copy has its own inputs


def test_single_rank_needs_no_process_group():
    b = _bench()
    assert b.max_over_ranks(3.5, 1, torch.device("cpu")) == 3.5
    assert b.job_rate(7.0, 1, torch.device("cpu")) == 7.0
