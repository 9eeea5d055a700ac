"""The multi-rank benchmark path on the CPU: two gloo ranks, each timing its
own replica; the job time is the maximum over ranks and the job throughput
counts every rank's work (weak scaling). No GPU and no data-path collective:
the attention path shards into independent (b, h, row-block) problems."""

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = [12.5, 17.0][rank]  # the second rank is slower
        job = bench.max_over_ranks(ms, dist, "cpu")
        q.put((rank, job, bench.job_throughput(world, 2.0e12, job)))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_throughput_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    for rank, job, tput in res:
        assert job == 17.0                       # every rank sees the slowest rank's time
        assert tput == pytest.approx(2 * 2.0e12 / 17.0e-3 / 1e12)


def test_single_process_is_identity():
    assert bench.max_over_ranks(3.5) == 3.5
    assert bench.job_throughput(1, 1e12, 1000.0) == pytest.approx(1.0)
