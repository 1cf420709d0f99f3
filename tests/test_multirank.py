"""Host-side logic of multi-GPU runs, on CPU with the gloo backend (2 ranks).

The path shards by (batch, kv head) units with no exchange step, so a run on
N GPUs is N independent replicas; the only cross-rank step is the max over
ranks of the timed region. These tests run that step with real processes.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import synth


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = [3.0, 7.5][rank]
        mx = bench.max_over_ranks(ms, world)
        value = bench.job_throughput(1000, world, mx)
        w = bench.replica_workload(synth.WORKLOADS[1], rank)
        out[rank] = (mx, value, w.seed)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_throughput_with_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        mp.start_processes(_worker, args=(2, _free_port(), out), nprocs=2, join=True, start_method="spawn")
        res = dict(out)
    assert res[0][0] == res[1][0] == 7.5
    assert res[0][1] == res[1][1] == pytest.approx(2 * 1000 / 7.5e-3)
    assert res[0][2] != res[1][2]  # replicas draw independent problems


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(4.0, 1) == 4.0
    assert bench.job_throughput(32768, 1, 2.0) == pytest.approx(32768 / 2e-3)


def _worker_dies(rank, world, port, out):
    """Rank 1 leaves before the timing reduction (as a rank that failed between steps would);
    rank 0 must get an error from its collective within the process-group timeout, not hang."""
    import datetime
    import time

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=5))
    if rank == 1:
        out[1] = "left"
        return  # no collective, no destroy: the process simply ends
    t0 = time.time()
    try:
        bench.max_over_ranks(1.0, world)
        out[0] = ("no error", time.time() - t0)
    except Exception as ex:  # gloo reports the lost peer or the timeout
        out[0] = (type(ex).__name__, time.time() - t0)


def test_a_rank_that_leaves_makes_the_others_fail_fast():
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        procs = mp.start_processes(_worker_dies, args=(2, _free_port(), out), nprocs=2, join=False,
                                   start_method="spawn")
        for p in procs.processes:
            p.join(60)
        res = dict(out)
        for p in procs.processes:
            if p.is_alive():
                p.kill()
    assert res.get(1) == "left"
    kind, took = res[0]
    assert kind != "no error"
    assert took < 30.0
