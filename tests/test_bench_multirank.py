"""The N > 1 path of bench.py on CPU: two gloo ranks run the same reduction
steps the GPU ranks run over NCCL (max over ranks of the step time, whole-job
throughput), and the reference arm prints on rank 0 only."""
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
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        ms = [1.5, 2.25][rank]           # per-rank step times
        m = bench.max_over_ranks(ms, dist, torch.device("cpu"))
        v = bench.job_tflops(world, 1e12, m)
        out[rank] = (m, v)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_rank_reduction_takes_the_slowest_rank():
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(_rank_main, args=(2, _free_port(), out), nprocs=2, join=True, start_method="spawn")
        res = dict(out)
    assert res[0] == res[1]
    m, v = res[0]
    assert m == 2.25                                  # max over ranks, not the mean or rank 0's own
    assert v == pytest.approx(2 * 1e12 / 2.25e-3 / 1e12)   # both ranks' work over the slowest time


def test_reference_arm_other_ranks_print_nothing():
    class A:
        warmup, steps, gpus = 1, 1, 2
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        bench.reference_arm(A(), rank=1)
    assert buf.getvalue() == ""
