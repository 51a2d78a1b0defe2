"""Multi-rank bookkeeping of bench.py, on CPU with two gloo ranks.

Each rank runs its own replica of the workload (the (batch, head) problems are
independent, so there is no collective on the data path).  The timing is the
maximum over ranks, the value counts the work of every rank, and only rank 0
runs and prints the oracle's reference arm.
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
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        # the slowest rank's time wins
        m = bench.max_over_ranks(10.0 + 5.0 * rank)
        # the reference arm: rank 0 only (the others exit without work)
        class A:
            steps = 1
            warmup = 0
            workload_desc = "test"
        from differentiable_sparse_attention_b200 import workloads as W
        ref = bench.run_reference(A, [W.TINY_FP32.with_(N=64)], rank, world)
        out[rank] = (m, ref is None)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_reference_gating():
    world = 2
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    assert out[0][0] == 15.0 and out[1][0] == 15.0
    assert out[0][1] is False      # rank 0 ran the oracle sample
    assert out[1][1] is True       # rank 1 did no work


def test_whole_job_value_counts_every_rank():
    import bench
    # 2 ranks, each 3 steps of 1e12 effective FLOP, slowest rank 1500 ms in total
    assert bench.whole_job_tflops(1e12, 3, 2, 1500.0) == pytest.approx(4.0)
    # one rank alone on the same work and time: half the job
    assert bench.whole_job_tflops(1e12, 3, 1, 1500.0) == pytest.approx(2.0)


def test_max_over_ranks_without_group():
    import bench
    assert not dist.is_initialized()
    assert bench.max_over_ranks(3.5) == 3.5
