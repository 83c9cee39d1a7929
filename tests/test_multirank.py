"""Multi-process host logic of the bench on CPU (gloo, world size 2): one
independent sequence per rank, the slowest rank's time, the whole-job value.
No GPU is used."""

import datetime
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        from compressed_sparse_long_compress_b200 import workloads as W
        # each rank times a different step length; every rank must see the max
        ms = bench.max_over_ranks(2.0 + rank, world)
        bench.barrier(world)
        wl = W.WORKLOADS["tiny"]
        x = W.prefill_inputs(wl.csa, bench.rank_seed(wl.wid, rank), with_indexer=False)
        out[rank] = (ms, float(x["q"].float().sum()), bench.job_value(4096, ms, world))
    finally:
        dist.destroy_process_group()


def test_two_ranks_max_time_independent_inputs_and_job_value():
    world = 2
    out = mp.Manager().dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    ms0, q0, v0 = out[0]
    ms1, q1, v1 = out[1]
    assert ms0 == ms1 == 3.0                      # max over ranks, on every rank
    assert q0 != q1                               # each rank its own seeded sequence
    assert v0 == v1 == pytest.approx(2 * 4096 / 3e-3)   # all ranks' tokens / slowest time


def test_single_rank_helpers_without_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(1.25, 1) == 1.25
    assert bench.rank_seed(2, 0) == 2 and bench.rank_seed(2, 3) == 32
    assert bench.job_value(65536, 10.0, 1) == pytest.approx(6553600.0)


def test_reference_arm_runs_on_rank_zero_only(capsys):
    sys.path.insert(0, ROOT)
    import argparse
    import bench
    args = argparse.Namespace(workload="tiny", steps=1, warmup=0, gpus=2)
    bench.run_reference(args, world=2, rank=1)     # other ranks exit without work or output
    assert capsys.readouterr().out == ""
