"""The multi-GPU plumbing of bench.py on CPU: two gloo ranks, world size 2.

The path shards by independent video streams, with no data-path collective:
each rank draws its own stream (same shapes, different seed), the step time is
the max over ranks, and the whole-job figure divides it by the chunks all
ranks processed."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import lcsa_inputs as li


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        w = bench.rank_workload(li.workload("tiny"), rank)
        x = li.make_inputs(w)
        local_ms = 1.0 + rank  # rank 1 is the slower one
        bench.barrier(world)
        worst = bench.max_over_ranks(local_ms, world, device="cpu")
        q_sum = float(x["q"].float().sum())
        out[rank] = (w.seed, tuple(x["q"].shape), q_sum, worst,
                     bench.whole_job_ms_per_chunk(worst, 1, world))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_weak_scaling_bookkeeping():
    world = 2
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    r0, r1 = out[0], out[1]
    assert r0[0] != r1[0]                 # independent streams
    assert r0[1] == r1[1]                 # of the same shape
    assert r0[2] != r1[2]                 # and different content
    assert r0[3] == r1[3] == 2.0          # every rank sees the slowest rank's time
    assert r0[4] == r1[4] == 1.0          # 2 chunks in 2 ms


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.whole_job_ms_per_chunk(26.0, 13, 1) == 2.0
    w = li.workload("chunk")
    assert bench.rank_workload(w, 0).seed == w.seed
    assert bench.rank_workload(w, 3).seed == w.seed + 3000
