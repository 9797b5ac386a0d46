"""Multi-GPU bookkeeping on CPU ranks: two gloo processes stand in for two replicas and
check that the timing is the maximum over ranks, that the whole-job throughput counts every
replica's work, and that replicas draw different data (no GPU involved)."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from padded_variable_length_b200 import replicas as R
from padded_variable_length_b200 import workloads as W


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        my_ms = 10.0 + 5.0 * rank  # rank 1 is the slow one
        mx = R.max_over_ranks(my_ms, torch.device("cpu"))
        value = R.job_throughput(world, 2.0e12, 4, mx)
        w = W.config(1)
        w.seed = R.replica_seed(w.seed, rank)
        q = W.tensors(w, with_grad=False)["q"]
        out[rank] = (mx, value, float(q.float().sum()))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks():
    world, port = 2, _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_rank_main, args=(world, port, out), nprocs=world, join=True,
                       start_method="spawn")
    (mx0, v0, s0), (mx1, v1, s1) = out[0], out[1]
    assert mx0 == mx1 == 15.0                      # the slowest rank's time, on every rank
    assert v0 == v1 == pytest.approx(2 * 2.0e12 * 4 / 15e-3 / 1e12)
    assert s0 != s1                                # each replica its own data


def test_single_process_is_identity():
    assert R.max_over_ranks(3.5) == 3.5
    assert R.job_throughput(1, 1.0e12, 1, 1000.0) == pytest.approx(1.0)
    with pytest.raises(ValueError):
        R.job_throughput(1, 1.0, 1, 0.0)
    assert R.replica_seed(1002, 0) == 1002
