"""Host side of the multi-GPU benchmark path, run as two gloo processes on the
CPU.  The scan shards by (b, h): every rank runs its own replica of the
workload and no data-path collective exists; what the ranks share is the
timing protocol (barriers around the timed region, the slowest rank's time,
the whole-job throughput), which is what is checked here."""
import datetime
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench

WORLD = 2


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, port, ms_by_rank, units, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=WORLD, timeout=datetime.timedelta(seconds=60))
    try:
        dist.barrier()
        ms = bench.max_over_ranks(torch, dist, ms_by_rank[rank], torch.device("cpu"))
        value = bench.whole_job_value(WORLD, units, ms)
        # a rank that sits out (no bench work) still takes part in the same collectives
        dist.barrier()
        q.put((rank, ms, value))
    finally:
        dist.destroy_process_group()


def test_two_ranks_agree_on_slowest_time_and_value():
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    ms_by_rank = [1.25, 1.75]
    units = 393_120
    procs = [ctx.Process(target=_worker, args=(r, port, ms_by_rank, units, q)) for r in range(WORLD)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    results = sorted(q.get(timeout=10) for _ in range(WORLD))
    for rank, ms, value in results:
        assert ms == pytest.approx(max(ms_by_rank))
        assert value == pytest.approx(WORLD * units / (max(ms_by_rank) * 1e-3) / 1e6)


def test_single_rank_needs_no_collective():
    assert bench.max_over_ranks(torch, None, 2.5, torch.device("cpu")) == 2.5
    assert bench.whole_job_value(1, 1_000_000, 1.0) == pytest.approx(1000.0)
