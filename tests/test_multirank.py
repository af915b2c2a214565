"""Multi-process host logic of bench.py on CPU: two gloo ranks (replicas).

The layer's work splits by sequence and head with no exchange, so N GPUs run N
independent replicas; what crosses ranks is only the timing: every rank gets the
maximum step time over the ranks, the job rate is all ranks' units over that time,
and the reference arm runs on rank 0 alone.
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


def _rank_main(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    try:
        # rank r took 1 + r ms per step and 0.5 + 2 r ms in its prefill call
        ms, pms = bench.max_over_ranks(torch, [1.0 + rank, 0.5 + 2.0 * rank], torch.device("cpu"))
        rate = bench.job_rate(world, 4096, ms)

        class A:
            steps, warmup = 1, 1
        ref = bench.bench_reference(A(), rank, world) if rank != 0 else "rank0"
        out[rank] = (ms, pms, rate, ref)
    finally:
        dist.destroy_process_group()


def test_two_replicas_take_the_slowest_rank():
    world = 2
    port = _free_port()
    mgr = mp.Manager()
    out = mgr.dict()
    mp.start_processes(_rank_main, args=(world, port, out), nprocs=world, join=True, start_method="spawn")
    for r in range(world):
        ms, pms, rate, ref = out[r]
        assert ms == pytest.approx(2.0)          # max of 1 and 2 ms
        assert pms == pytest.approx(2.5)         # max of 0.5 and 2.5 ms
        assert rate == pytest.approx(2 * 4096 / 2e-3)
    assert out[1][3] is None                     # the reference arm prints on rank 0 only


def test_job_rate_single_rank():
    import bench
    assert bench.job_rate(1, 4096, 0.5) == pytest.approx(4096 / 0.5e-3)
