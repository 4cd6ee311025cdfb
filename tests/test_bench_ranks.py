"""The multi-rank plumbing of bench.py on the CPU: two gloo ranks agree on the slowest
rank's time, the whole-job rate counts every rank's shard, shards are distinct, and the
reference arm prints from rank 0 only."""

import contextlib
import io
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    dist.init_process_group("gloo", init_method="tcp://127.0.0.1:%d" % port, rank=rank, world_size=world)
    try:
        # per-rank step times: the slowest rank (rank 1) sets the step
        ms = bench.max_over_ranks(1.0 + rank, world, dist, "cpu")
        rate = bench.whole_job_rate(65536, world, ms)
        out[rank] = (ms, rate, bench.shard_seed(rank))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks():
    world = 2
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_rank_main, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    assert res[0][0] == res[1][0] == 2.0  # both ranks see the slowest rank's time
    assert res[0][1] == res[1][1] == pytest.approx(2 * 65536 / 2.0e-3)  # all shards over that time
    assert res[0][2] != res[1][2]  # distinct input shards


def test_single_rank_is_identity():
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.whole_job_rate(1000, 1, 2.0) == pytest.approx(5.0e5)


def test_reference_arm_prints_on_rank_zero_only():
    class A:
        steps, warmup = 1, 3
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        bench.run_reference(A(), 1, 2)
    assert buf.getvalue() == ""
