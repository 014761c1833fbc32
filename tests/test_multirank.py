"""CPU tests of the multi-process bench plumbing with two gloo ranks.

Each rank decodes its own independent batch (no collective on the data path); the
only exchanges are the timing reductions: the job time is the slowest rank's and
the work is the sum over ranks.
"""
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


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        t, u = bench.reduce_max_sum(10.0 * (rank + 1), 100.0 + rank, torch.device("cpu"))
        bench.barrier()
        q.put((rank, t, u, bench.rank_seed(2, rank)))
    finally:
        dist.destroy_process_group()


def test_two_rank_time_is_max_and_units_are_summed():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, t, u, seed in res:
        assert t == 20.0          # max over ranks
        assert u == 201.0         # sum over ranks
    assert res[0][3] != res[1][3]  # independent batches per rank
    assert res[0][3] == 1002       # rank 0 runs the workload's own seed


def test_single_process_reduction_is_identity():
    assert bench.reduce_max_sum(3.5, 7.0, torch.device("cpu")) == (3.5, 7.0)


def test_reference_arm_runs_on_rank0_only(monkeypatch, capsys):
    import sys
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setattr(sys, "argv", ["bench.py", "--impl", "reference", "--steps", "3", "--warmup", "3"])
    bench.main()
    assert capsys.readouterr().out == ""
