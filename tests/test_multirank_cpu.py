"""Host logic of the multi-rank benchmark on CPU: two gloo ranks, no GPU.

Every (batch, head) sequence of the recurrence is independent, so N GPUs run N
independent batches and no collective touches the data path. What the ranks do
share is the timing: each reports its own step time and the job uses the
slowest, and the whole-job throughput counts every rank's tokens.
"""
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


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import bench
    import lattice_inputs as LI
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        mine = 10.0 + 5.0 * rank  # rank 1 is the slow one
        got = bench.max_over_ranks(torch, dist, mine, torch.device("cpu"))
        w0 = LI.WORKLOADS["small_train"]
        wr = bench.rank_workload(w0, rank)
        out[rank] = (got, wr.seed, bench.job_tokens_per_s(world, wr, got))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_time_and_count_all_tokens():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(_worker, args=(world, port, out), nprocs=world, join=True,
                           start_method="spawn")
        res = dict(out)
    assert res[0][0] == res[1][0] == 15.0
    assert res[0][1] != res[1][1], "each rank draws its own batch"
    import lattice_inputs as LI
    w = LI.WORKLOADS["small_train"]
    assert res[0][2] == pytest.approx(2 * w.B * w.T / 15e-3)


def test_single_process_needs_no_group():
    import bench
    assert bench.max_over_ranks(torch, None, 3.5, torch.device("cpu")) == 3.5


def test_reference_arm_other_ranks_exit_without_work(monkeypatch):
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setattr(sys, "argv", ["bench.py", "--impl", "reference", "--gpus", "2"])
    assert bench.main() == 0
