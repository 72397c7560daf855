"""The multi-GPU plumbing of bench.py on CPU: two gloo ranks, world size 2.

The path shards by independent video streams, with no data-path collective:
each rank draws its own stream (same shapes, different seed), the step time is
the max over ranks, and the whole-job figure divides it by the chunks all
ranks processed."""
import os
import socket

import numpy as np
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


# --------------------------------------------------------------- head split
def test_rank_units_cover_every_unit_once_streams_first():
    from block_sparse_causal_lcsa_b200.partition import rank_slices, rank_units
    for B in (1, 2, 3, 4, 5, 8):
        for H in (1, 3, 12):
            for world in (1, 2, 3, 4, 8):
                shares = [rank_units(B, H, world, r) for r in range(world)]
                flat = [u for s in shares for u in s]
                assert flat == [(b, h) for b in range(B) for h in range(H)]   # each once, in order
                sizes = [len(s) for s in shares]
                assert max(sizes) - min(sizes) <= 1
                if B % world == 0:                                           # whole streams per rank
                    for r, s in enumerate(rank_slices(B, H, world, r) for r in range(world)):
                        assert all(h0 == 0 and h1 == H for _, h0, h1 in s)
                        assert len(s) == B // world
                for r in range(world):
                    sl = rank_slices(B, H, world, r)
                    assert sum(h1 - h0 for _, h0, h1 in sl) == sizes[r]
                    assert len(sl) <= -(-B // world) + 1
    # 12 heads of one stream over 8 ranks: heads split 1 or 2 per rank
    assert [rank_slices(1, 12, 8, r) for r in (0, 1)] == [[(0, 0, 1)], [(0, 1, 3)]]
    with pytest.raises(ValueError):
        rank_units(1, 12, 2, 2)


def _oracle_units(w, x, units):
    from oracle import lcsa_oracle as orc
    out = {}
    for b, h in units:
        ref = orc.lcsa_head(orc.widen(x["q"][b, h]), orc.widen(x["k"][b][h]), orc.widen(x["v"][b][h]),
                            top_k=w.top_k, density=w.density, window=w.window, mode=w.window_mode)
        out[(b, h)] = (ref["O"], ref["LSE"], [s.tolist() for s in ref["sel"]])
    return out


_PART_W = li.Workload("part", B=3, H=3, D=64, Y=16, X=16, q_frames=2, kv_past=(2, 4, 3), cap_frames=6,
                      density=0.3, seed=5)


def _partition_rank(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    from block_sparse_causal_lcsa_b200.partition import rank_units
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        x = li.make_inputs(_PART_W)
        mine = _oracle_units(_PART_W, x, rank_units(_PART_W.B, _PART_W.H, world, rank))
        parts = [None] * world
        dist.all_gather_object(parts, mine)        # test bookkeeping only: the path itself exchanges nothing
        if rank == 0:
            out["parts"] = parts
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_head_split_union_equals_single_rank():
    """Three ragged streams x 3 heads over 2 ranks (one stream is split by
    heads): each rank runs the oracle on its own units only; the union of the
    two shares is every unit exactly once, equal to the single-rank result."""
    world = 2
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_partition_rank, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(180)
        assert p.exitcode == 0
    parts = out["parts"]
    assert set(parts[0]).isdisjoint(parts[1])
    union = {**parts[0], **parts[1]}
    single = _oracle_units(_PART_W, li.make_inputs(_PART_W),
                           [(b, h) for b in range(_PART_W.B) for h in range(_PART_W.H)])
    assert set(union) == set(single)
    assert len(parts[0]) == len(parts[1]) + 1 or len(parts[1]) == len(parts[0]) + 1
    for key, (o, lse, sel) in single.items():
        go, glse, gsel = union[key]
        assert gsel == sel
        assert np.array_equal(go, o) and np.array_equal(glse, lse)
