"""The replica path of bench.py with two ranks on CPU (gloo): per-rank batches, the slowest rank's
time, the sum of all ranks' work, and the reference arm running on rank 0 alone."""
import argparse
import datetime
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _reduce_worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        ms, flops = bench.reduce_over_ranks(dist, torch, "cpu", 1.0 + rank, 10.0 * (rank + 1), world)
        e2e, _ = bench.reduce_over_ranks(dist, torch, "cpu", 5.0 - rank, 0.0, world)
        out[rank] = (ms, flops, e2e)
    finally:
        dist.destroy_process_group()


def test_replicas_take_the_slowest_rank_and_the_work_of_all():
    world, port = 2, _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_reduce_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    # every rank sees the same reduction: max of (1, 2) ms, sum of (10, 20) flops, max of (5, 4) ms
    assert res[0] == res[1] == (2.0, 30.0, 5.0)


def test_single_rank_is_unchanged():
    assert bench.reduce_over_ranks(None, torch, "cpu", 3.5, 7.0, 1) == (3.5, 7.0)


def test_each_replica_draws_its_own_batch_of_the_same_size():
    a, b = bench.rank_workload("packed", 0, 0), bench.rank_workload("packed", 0, 1)
    assert a.total == b.total == 16384 and a.heads == b.heads and a.cp == b.cp
    assert list(a.cu_seqlens) != list(b.cu_seqlens)
    # the long document is the same on every rank
    assert list(bench.rank_workload("long_doc", 0, 3).cu_seqlens) == [0, 65536]


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    monkeypatch.setenv("RANK", "1")
    bench.run_reference(argparse.Namespace(seed=0, steps=1, warmup=0, gpus=2))
    assert capsys.readouterr().out == ""
