"""GPU parity: the CUDA path through the C ABI against the fp64 oracle.

Pooled features and block selections must match bit for bit; attention output
must be within max-abs 2e-2 and relative L2 1e-2 of the fp64 result (bf16
inputs, fp32 accumulation). Small variants of every workload are compared on
every row; the full-size workloads are compared on every selection row and on
sampled query blocks of O.
"""
import numpy as np
import pytest
import torch

import lcsa_inputs as li
from oracle import lcsa_oracle as orc

from lcsa_harness import (build_cache, check_output, check_selection, compare_all, oracle_head,
                          params_of, ring_to_logical, run_gpu)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lc():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import block_sparse_causal_lcsa_b200 as m
    return m


SMALL = [
    li.workload("tiny"),
    li.small_variant(li.workload("chunk"), H=2, Y=24, X=40),
    li.small_variant(li.workload("multistream"), H=2, Y=16, X=24),
    li.small_variant(li.workload("uhr_truncate"), H=2, Y=48, X=56, window=3),
    li.small_variant(li.workload("uhr_preserve"), H=2, Y=48, X=56, window=3),
    li.small_variant(li.workload("clip_5"), H=1, Y=16, X=24),
    li.small_variant(li.workload("clip"), H=1, Y=16, X=24),
    li.small_variant(li.workload("clip_30"), H=1, Y=16, X=24),
    li.small_variant(li.workload("tiny"), H=1, Y=16, X=16, D=128, kv_past=(4,), cap_frames=6),
]


@pytest.mark.parametrize("w", SMALL, ids=[w.name for w in SMALL])
def test_small_workloads_every_row(lc, w):
    x = li.make_inputs(w)
    g = run_gpu(lc, w, x)
    assert g["err"] == 0
    compare_all(w, x, g)


FULL = ["chunk", "multistream", "uhr_truncate", "uhr_preserve"]
# workloads whose O is compared on every query block of the checked heads (the
# oracle does 66 query blocks of a 768x1408 head in seconds); the 1536x2688
# ones on 8 sampled query blocks
FULL_O_ALL_ROWS = {"chunk", "multistream"}


@pytest.mark.parametrize("name", FULL)
def test_full_size_selection_all_rows_output_checked(lc, name):
    w = li.workload(name)
    x = li.make_inputs(w)
    g = run_gpu(lc, w, x)
    assert g["err"] == 0
    rng = np.random.default_rng(11)
    nQB = g["blk_cnt"].shape[2]
    if name in FULL_O_ALL_ROWS:
        rows = list(range(nQB))
    else:
        rows = sorted(rng.choice(nQB, size=6, replace=False).tolist() + [0, nQB - 1])
    heads = [0, w.H - 1]
    for b in range(w.B):
        for h in range(w.H):
            ref = oracle_head(w, x, b, h, rows=rows if h in heads else [])
            where = "%s b%d h%d" % (name, b, h)
            assert np.array_equal(g["q_pool"][b, h].reshape(-1, w.D), ref["q_pool"]), where
            assert np.array_equal(ring_to_logical(g["cache"], g["k_pool_ring"], b, h), ref["k_pool"]), where
            check_selection(g["blk_idx"][b, h], g["blk_cnt"][b, h], ref["sel"], where)
            if h in heads:
                check_output(g["O"][b, h], ref["O"], g["LSE"][b, h], ref["LSE"], where)


@pytest.mark.parametrize("name", ["clip_5", "clip", "clip_30"])
def test_full_clip_selection_and_sampled_output(lc, name):
    """The whole 101-frame clip at each density of the sweep (5%, 13.6%, 30%):
    pooled features and every selection row of every head bit for bit; O and
    LSE of two heads on sampled query blocks, the newest frame pair's (the
    longest rows: 43, 117 and 258 kept blocks) among them."""
    w = li.workload(name)
    x = li.make_inputs(w)
    dev = "cuda"
    k = x["k"][0].unsqueeze(0).to(dev)
    v = x["v"][0].unsqueeze(0).to(dev)
    q = x["q"].to(dev)
    q_pool, k_pool = lc.pool_qk(q, k)
    cache = lc.KVCache.wrap(k, v, k_pool)
    params = params_of(lc, w)
    idx, cnt = lc.select_blocks(q_pool, w.q_frames, cache, params)
    o, lse = lc.sparse_attn_fwd(q, cache, idx, cnt, workspace=lc.attn_workspace(w.D))
    torch.cuda.synchronize()
    assert lc.last_device_error() == 0
    idx, cnt = idx.cpu().numpy(), cnt.cpu().numpy()
    O, L = o.double().cpu().numpy(), lse.double().cpu().numpy()
    qp, kp = q_pool.cpu().numpy(), k_pool.cpu().numpy()
    nQB = cnt.shape[2]
    HbWb = w.Hb * w.Wb
    rows = [0, 65, 400, nQB - HbWb, nQB - HbWb // 2, nQB - 1]
    longest = int(np.ceil(w.density * nQB))
    for h in range(w.H):
        qh, kh = orc.widen(x["q"][0, h]), orc.widen(x["k"][0][h])
        rq, rk = orc.pool_blocks(qh), orc.pool_blocks(kh)
        assert np.array_equal(qp[0, h].reshape(-1, w.D), rq) and np.array_equal(kp[0, h].reshape(-1, w.D), rk)
        sel, Ks, Cs = orc.select_head(rq, rk, w.q_frames, w.q_frames, w.Y, w.X, density=w.density)
        check_selection(idx[0, h], cnt[0, h], sel, "%s h%d" % (name, h))
        assert int(cnt[0, h, nQB - 1]) == longest
        if h in (0, 7):
            ro, rl = orc.attend_head(qh, kh, orc.widen(x["v"][0][h]), sel, rows)
            check_output(O[0, h], ro, L[0, h], rl, "%s h%d" % (name, h))


@pytest.mark.parametrize("past", [250, 372])
def test_long_cache_many_candidates(lc, past):
    """A long cache: 756 and 1122 causal candidates per query block, so the
    top-K keeps 32 and 64 keys per lane in registers."""
    w = li.Workload("long", B=1, H=2, D=128, Y=16, X=24, q_frames=2, kv_past=(past,),
                    cap_frames=past + 2, density=0.05, seed=71)
    x = li.make_inputs(w)
    g = run_gpu(lc, w, x)
    assert g["err"] == 0
    compare_all(w, x, g)


def test_attention_on_oracle_mask(lc):
    """O computed from the oracle's own block lists (selection errors excluded)."""
    w = li.small_variant(li.workload("chunk"), H=2, Y=24, X=40)
    x = li.make_inputs(w)
    g = run_gpu(lc, w, x)
    step = g["step"]
    kmax = step.blk_idx.shape[-1]
    idx = np.full(step.blk_idx.shape, -1, np.int32)
    cnt = np.zeros(step.blk_cnt.shape, np.int32)
    refs = {}
    for h in range(w.H):
        ref = oracle_head(w, x, 0, h)
        refs[h] = ref
        for i, s in enumerate(ref["sel"]):
            s = s[::-1]  # any order of the kept blocks gives the same output
            idx[0, h, i, :len(s)] = s
            cnt[0, h, i] = len(s)
    o, lse = lc.sparse_attn_fwd(g["q"], g["cache"], torch.from_numpy(idx).cuda(),
                                torch.from_numpy(cnt).cuda())
    torch.cuda.synchronize()
    assert lc.last_device_error() == 0 and kmax == idx.shape[-1]
    for h in range(w.H):
        check_output(o[0, h].double().cpu().numpy(), refs[h]["O"], lse[0, h].double().cpu().numpy(),
                     refs[h]["LSE"], "h%d" % h)


def test_streaming_sequence_with_eviction(lc):
    """Five 2-frame chunks through a 6-frame cache; every step against the
    oracle applied to the concatenated, evicted timeline."""
    w = li.Workload("stream", B=1, H=2, D=128, Y=16, X=24, q_frames=2, kv_past=(8,),
                    cap_frames=6, density=0.4, seed=21)
    x = li.make_inputs(w)
    dev = "cuda"
    cache = lc.KVCache(1, w.H, w.cap_frames, w.Y, w.X, w.D, device=dev)
    step = lc.StreamingStep(cache, 2, params_of(lc, w))
    F = x["k"][0].shape[1]
    for s0 in range(0, F, 2):
        kc = x["k"][0][:, s0:s0 + 2].unsqueeze(0).to(dev)
        vc = x["v"][0][:, s0:s0 + 2].unsqueeze(0).to(dev)
        qc = torch.randn((1, w.H, 2, w.Y, w.X, w.D), generator=torch.Generator().manual_seed(s0)).to(torch.bfloat16)
        o, lse = step(qc.to(dev), kc, vc)
        torch.cuda.synchronize()
        assert lc.last_device_error() == 0
        lo = max(0, s0 + 2 - w.cap_frames)
        assert cache.state() == [(lo, s0 + 2)]
        for h in range(w.H):
            kt = orc.widen(x["k"][0][h, lo:s0 + 2])
            vt = orc.widen(x["v"][0][h, lo:s0 + 2])
            ref = orc.lcsa_head(orc.widen(qc[0, h]), kt, vt, density=w.density)
            assert np.array_equal(ring_to_logical(cache, cache.k_pool.cpu().numpy(), 0, h), ref["k_pool"])
            kc_ring = cache.k[0, h].cpu()
            for f in range(lo, s0 + 2):
                assert torch.equal(kc_ring[f % w.cap_frames], x["k"][0][h, f])
            check_selection(step.blk_idx[0, h].cpu().numpy(), step.blk_cnt[0, h].cpu().numpy(), ref["sel"])
            check_output(o[0, h].double().cpu().numpy(), ref["O"], lse[0, h].double().cpu().numpy(), ref["LSE"])


def test_tail_split_matches_unsplit_and_oracle(lc):
    """12 heads x 42 query blocks = 504 CTAs: on 148 SMs the last 60 query
    blocks run as split halves merged by a second kernel. Same selections,
    outputs within bf16 rounding of the unsplit kernel, and the oracle's."""
    w = li.small_variant(li.workload("chunk"), H=12, Y=48, X=56)
    x = li.make_inputs(w)
    g = run_gpu(lc, w, x)                      # the streaming step passes a workspace
    assert g["err"] == 0
    o2, l2 = lc.sparse_attn_fwd(g["q"], g["cache"], g["step"].blk_idx, g["step"].blk_cnt)   # unsplit
    torch.cuda.synchronize()
    assert lc.last_device_error() == 0
    o2, l2 = o2.double().cpu().numpy(), l2.double().cpu().numpy()
    assert np.abs(g["O"] - o2).max() <= 2.0 ** -7 * max(1.0, np.abs(o2).max())
    assert np.abs(g["LSE"] - l2).max() <= 1e-4
    compare_all(w, x, g, heads=[0, 5, 11])


def test_ingest_chunk_equals_pool_then_append(lc):
    """One launch for Q pooling and the fused K/V append gives the same q_pool
    and cache as pool_qk followed by kv_append, bit for bit (two streams, an
    odd first chunk, then a wrapped ring)."""
    H, Y, X, D, cap = 2, 16, 24, 128, 4
    a = lc.KVCache(2, H, cap, Y, X, D)
    b = lc.KVCache(2, H, cap, Y, X, D)
    for c in (a, b):
        c.k.zero_(), c.v.zero_(), c.k_pool.zero_()
    g = torch.Generator().manual_seed(17)
    for t in (3, 2, 2, 2):
        q, k, v = (torch.randn((2, H, t, Y, X, D), generator=g).to(torch.bfloat16).cuda() for _ in range(3))
        qp_a = lc.ingest_chunk(q, a, k, v)
        qp_b = lc.pool_qk(q)[0]
        lc.kv_append(b, k, v)
        torch.cuda.synchronize()
        assert torch.equal(qp_a, qp_b) and a.state() == b.state()
    assert lc.last_device_error() == 0
    assert torch.equal(a.k, b.k) and torch.equal(a.v, b.v) and torch.equal(a.k_pool, b.k_pool)


def test_graph_replay_equals_eager_steps(lc):
    """Eight 2-frame chunks through a 6-frame cache, eagerly and from CUDA graphs
    (one per ring phase): identical outputs, cache contents and state."""
    w = li.Workload("graph", B=2, H=2, D=128, Y=16, X=24, q_frames=2, kv_past=(0, 0), cap_frames=6,
                    density=0.4, seed=91)
    caches = [lc.KVCache(w.B, w.H, w.cap_frames, w.Y, w.X, w.D) for _ in range(2)]
    for c in caches:
        c.k.zero_(), c.v.zero_(), c.k_pool.zero_()
    steps = [lc.StreamingStep(c, 2, params_of(lc, w)) for c in caches]
    g = torch.Generator().manual_seed(7)
    for t in range(8):
        q, k, v = (torch.randn((w.B, w.H, 2, w.Y, w.X, w.D), generator=g).to(torch.bfloat16).cuda() for _ in range(3))
        o0, l0 = steps[0](q, k, v)
        o1, l1 = steps[1].graph_step(q, k, v)
        torch.cuda.synchronize()
        assert lc.last_device_error() == 0
        assert torch.equal(o0, o1) and torch.equal(l0, l1), "step %d" % t
        assert caches[0].state() == caches[1].state()
    assert torch.equal(caches[0].k, caches[1].k) and torch.equal(caches[0].v, caches[1].v)
    assert torch.equal(caches[0].k_pool, caches[1].k_pool)
    # filling states (empty, 2, 4 frames), then the three phases of a full ring,
    # which steps 7 and 8 replay
    assert len(steps[1]._graphs) == 6


def test_host_pipeline_equals_eager_steps(lc):
    """Six chunks from pinned host memory through HostPipeline (copies on their
    own streams, two alternating input sets) against the same chunks stepped
    eagerly from device memory: identical outputs and cache contents."""
    w = li.Workload("hostpipe", B=1, H=2, D=128, Y=16, X=24, q_frames=2, kv_past=(0,), cap_frames=6,
                    density=0.4, seed=93)
    caches = [lc.KVCache(w.B, w.H, w.cap_frames, w.Y, w.X, w.D) for _ in range(2)]
    for c in caches:
        c.k.zero_(), c.v.zero_(), c.k_pool.zero_()
    steps = [lc.StreamingStep(c, 2, params_of(lc, w)) for c in caches]
    pipe = lc.HostPipeline(steps[1])
    g = torch.Generator().manual_seed(8)
    shp = (w.B, w.H, 2, w.Y, w.X, w.D)
    chunks = [tuple(torch.randn(shp, generator=g).to(torch.bfloat16).pin_memory() for _ in range(3))
              for _ in range(6)]
    outs = [torch.empty(shp, dtype=torch.bfloat16).pin_memory() for _ in range(6)]
    done = [pipe.submit(*c, outs[t]) for t, c in enumerate(chunks)]
    ref = []
    for c in chunks:
        o, _ = steps[0](*(t.cuda() for t in c))
        ref.append(o.cpu())
    done[-1].synchronize()
    torch.cuda.synchronize()
    assert lc.last_device_error() == 0
    for t in range(6):
        assert torch.equal(outs[t], ref[t]), "chunk %d" % t
    assert caches[0].state() == caches[1].state()
    assert torch.equal(caches[0].k, caches[1].k) and torch.equal(caches[0].v, caches[1].v)
    assert torch.equal(caches[0].k_pool, caches[1].k_pool)


def test_native_pipeline_equals_eager_steps(lc):
    """Six chunks from pinned host memory through the library's pipeline
    (lcsa_pipeline_*: uploads, step and read-back on its own streams) against
    the same chunks stepped eagerly from device memory: identical outputs,
    cache contents and cache state; the pipeline's timer covers the run."""
    w = li.Workload("nativepipe", B=2, H=2, D=128, Y=16, X=24, q_frames=2, kv_past=(0, 0), cap_frames=6,
                    density=0.4, seed=95)
    caches = [lc.KVCache(w.B, w.H, w.cap_frames, w.Y, w.X, w.D) for _ in range(2)]
    for c in caches:
        c.k.zero_(), c.v.zero_(), c.k_pool.zero_()
    step = lc.StreamingStep(caches[0], 2, params_of(lc, w))
    pipe = lc.NativePipeline(caches[1], 2, params_of(lc, w))
    g = torch.Generator().manual_seed(9)
    shp = (w.B, w.H, 2, w.Y, w.X, w.D)
    chunks = [tuple(torch.randn(shp, generator=g).to(torch.bfloat16).pin_memory() for _ in range(3))
              for _ in range(6)]
    outs = [torch.empty(shp, dtype=torch.bfloat16).pin_memory() for _ in range(6)]
    pipe.start_timer()
    for t, c in enumerate(chunks):
        pipe.submit(*c, outs[t])
    pipe.sync()
    assert pipe.elapsed_ms() > 0.0
    for t, c in enumerate(chunks):
        o, _ = step(*(x.cuda() for x in c))
        torch.cuda.synchronize()
        assert torch.equal(o.cpu(), outs[t]), "chunk %d" % t
    assert lc.last_device_error() == 0
    assert caches[0].state() == caches[1].state()
    assert torch.equal(caches[0].k, caches[1].k) and torch.equal(caches[0].v, caches[1].v)
    assert torch.equal(caches[0].k_pool, caches[1].k_pool)
    with pytest.raises(ValueError):
        pipe.submit(chunks[0][0].cuda(), *chunks[0][1:], outs[0])
    pipe.close()


def test_host_pipeline_rejects_device_and_pageable_tensors(lc):
    cache = lc.KVCache(1, 1, 4, 8, 8, 128)
    step = lc.StreamingStep(cache, 2, lc.SelectParams(top_k=1))
    pipe = lc.HostPipeline(step)
    shp = (1, 1, 2, 8, 8, 128)
    pinned = [torch.zeros(shp, dtype=torch.bfloat16).pin_memory() for _ in range(4)]
    with pytest.raises(ValueError):
        pipe.submit(pinned[0].cuda(), *pinned[1:])
    with pytest.raises(ValueError):
        pipe.submit(torch.zeros(shp, dtype=torch.bfloat16), *pinned[1:])


@pytest.mark.parametrize("first,q_frames", [(1, 1), (3, 3), (5, 2)])
def test_odd_first_chunk_partial_blocks(lc, first, q_frames):
    """A stream whose first chunk has an odd frame count: the oldest key block
    (and, for odd query counts, the oldest query block) holds one frame."""
    w = li.Workload("odd", B=1, H=2, D=128, Y=16, X=16, q_frames=q_frames, kv_past=(first - q_frames,),
                    cap_frames=8, density=0.5, seed=31 + first)
    x = li.make_inputs(w)
    dev = "cuda"
    cache = lc.KVCache(1, w.H, w.cap_frames, w.Y, w.X, w.D, device=dev)
    k = x["k"][0].unsqueeze(0).to(dev)
    v = x["v"][0].unsqueeze(0).to(dev)
    lc.kv_append(cache, k, v, lc.pool_qk(k)[0])
    assert cache.state() == [(1, first + 1)]
    q = x["q"].to(dev)
    qp = lc.pool_qk(q)[0]
    params = params_of(lc, w)
    idx, cnt = lc.select_blocks(qp, q_frames, cache, params)
    o, lse = lc.sparse_attn_fwd(q, cache, idx, cnt)
    torch.cuda.synchronize()
    assert lc.last_device_error() == 0
    for h in range(w.H):
        ref = oracle_head(w, x, 0, h)
        assert np.array_equal(qp[0, h].reshape(-1, w.D).cpu().numpy(), ref["q_pool"])
        assert np.array_equal(ring_to_logical(cache, cache.k_pool.cpu().numpy(), 0, h), ref["k_pool"])
        check_selection(idx[0, h].cpu().numpy(), cnt[0, h].cpu().numpy(), ref["sel"])
        check_output(o[0, h].double().cpu().numpy(), ref["O"], lse[0, h].double().cpu().numpy(), ref["LSE"])


@pytest.mark.parametrize("cap,chunks", [(8, (3, 2, 2, 2, 2)), (4, (5, 2, 6)), (6, (2, 10, 2)),
                                         (6, (1, 2, 2, 2))])
def test_fused_append_equals_pool_then_append(lc, cap, chunks):
    """kv_append without a pooled K (K pooled while it is copied) leaves the
    ring cache bit for bit as pool_qk followed by kv_append with the pooled K:
    odd first chunks, chunks longer than the cache, wrap-around."""
    H, Y, X, D = 2, 16, 24, 128
    g = torch.Generator().manual_seed(81 + cap)
    a = lc.KVCache(2, H, cap, Y, X, D)
    b = lc.KVCache(2, H, cap, Y, X, D)
    for c in (a, b):
        c.k.zero_(), c.v.zero_(), c.k_pool.zero_()
    timeline = [[None] * H for _ in range(2)]   # the oracle's cache of each (stream, head)
    for t in chunks:
        k_host = (torch.randn((2, H, t, Y, X, D), generator=g) * 3).to(torch.bfloat16)
        k = k_host.cuda()
        v = torch.randn((2, H, t, Y, X, D), generator=g).to(torch.bfloat16).cuda()
        lc.kv_append(a, k, v)
        lc.kv_append(b, k, v, lc.pool_qk(k)[0])
        assert a.state() == b.state()
        for s_ in range(2):
            for h in range(H):
                timeline[s_][h] = orc.kv_append(timeline[s_][h], orc.widen(k_host[s_, h]), cap)
    torch.cuda.synchronize()
    assert lc.last_device_error() == 0
    assert torch.equal(a.k, b.k) and torch.equal(a.v, b.v)
    assert torch.equal(a.k_pool, b.k_pool)
    # and the ring holds the oracle's cache, with the oracle's means of it as pooled rows
    for s_ in range(2):
        for h in range(H):
            lo, hi = a.state()[s_]
            frames = torch.stack([a.k[s_, h, f % cap].cpu() for f in range(lo, hi)])
            assert np.array_equal(frames.double().numpy(), timeline[s_][h])
            ref = orc.pool_blocks(timeline[s_][h])
            assert np.array_equal(ring_to_logical(a, a.k_pool.cpu().numpy(), s_, h), ref)


@pytest.mark.parametrize("kw", [dict(density=1.0), dict(top_k=1000), dict(top_k=1),
                                dict(density=0.3, window=99, window_mode=1)])
def test_degenerate_selection_parameters(lc, kw):
    w = li.Workload("edge", B=1, H=1, D=128, Y=16, X=24, q_frames=2, kv_past=(4,), cap_frames=6,
                    seed=41, **kw)
    x = li.make_inputs(w)
    g = run_gpu(lc, w, x)
    assert g["err"] == 0
    compare_all(w, x, g)


def test_planted_ties_resolve_to_lowest_index(lc):
    """Identical key blocks give exactly equal scores; the lowest ids win."""
    w = li.Workload("ties", B=1, H=1, D=128, Y=16, X=16, q_frames=2, kv_past=(4,), cap_frames=6,
                    top_k=3, seed=51)
    x = li.make_inputs(w)
    k = x["k"][0]
    for t in (0, 2, 4):  # every temporal block a copy of the first one
        k[:, t:t + 2] = k[:, 0:2]
    g = run_gpu(lc, w, x)
    compare_all(w, x, g)


def test_argument_errors_leave_outputs_untouched(lc):
    w = li.small_variant(li.workload("chunk"), H=1, Y=16, X=16)
    x = li.make_inputs(w)
    g = run_gpu(lc, w, x)
    step = g["step"]
    before = step.blk_idx.clone()
    with pytest.raises(lc.LcsaError) as e:
        lc.select_blocks(step.q_pool, 2, g["cache"], lc.SelectParams(density=0.5, window=4),
                         step.kmax, step.blk_idx, step.blk_cnt)
    assert e.value.status == -1
    # kmax = 1 cannot hold a full-density row: refused by the library
    idx1 = torch.full(step.blk_idx.shape[:3] + (1,), 5, dtype=torch.int32, device="cuda")
    cnt1 = torch.full(step.blk_cnt.shape, 5, dtype=torch.int32, device="cuda")
    with pytest.raises(lc.LcsaError) as e:
        lc.select_blocks(step.q_pool, 2, g["cache"], lc.SelectParams(density=1.0), 1, idx1, cnt1)
    assert e.value.status == -4
    # outputs whose row stride disagrees with kmax, or of the wrong type, are
    # refused by the binding before any launch
    with pytest.raises(ValueError):
        lc.select_blocks(step.q_pool, 2, g["cache"], lc.SelectParams(density=1.0), 1,
                         step.blk_idx, step.blk_cnt)
    with pytest.raises(ValueError):
        lc.select_blocks_noalloc(step.q_pool, 2, g["cache"], lc.SelectParams(density=0.5),
                                 step.blk_idx.long(), step.blk_cnt)
    torch.cuda.synchronize()
    assert torch.equal(before, step.blk_idx)
    assert (idx1 == 5).all() and (cnt1 == 5).all()


def test_wait_timeout_reports_and_context_survives(lc):
    """A wait that nothing completes gives up after its limit (no fault, no
    hang); the status reaches the host and the next calls still work."""
    assert lc.last_device_error() == 0
    lc.debug_stalled_wait(2_000_000)  # 2 ms
    assert lc.last_device_error() == -7
    assert lc.last_device_error() == 0  # cleared
    w = li.workload("tiny")
    x = li.make_inputs(w)
    g = run_gpu(lc, w, x)
    assert g["err"] == 0
    compare_all(w, x, g)


def test_out_of_range_block_id_is_reported(lc):
    w = li.workload("tiny")
    x = li.make_inputs(w)
    g = run_gpu(lc, w, x)
    step = g["step"]
    bad = step.blk_idx.clone()
    bad[0, 0, 0, 0] = 10_000
    lc.sparse_attn_fwd(g["q"], g["cache"], bad, step.blk_cnt)
    assert lc.last_device_error() == -8


def test_host_buffer_is_rejected_before_launch(lc):
    """A host-memory LSE buffer beside a chunk on the GPU: the binding raises
    ValueError before the library is called, and no device error follows."""
    w = li.workload("tiny")
    x = li.make_inputs(w)
    g = run_gpu(lc, w, x)
    step = g["step"]
    host_lse = torch.zeros(tuple(g["q"].shape[:5]), dtype=torch.float32)
    with pytest.raises(ValueError, match="lse must be a CUDA tensor"):
        lc.sparse_attn_fwd(g["q"], g["cache"], step.blk_idx, step.blk_cnt, lse=host_lse)
    assert lc.last_device_error() == 0


def test_exp2_polynomial_error_bound(lc):
    """The FMA-pipe 2^x that the softmax can use in place of the
    special-function unit stays within its fitted relative error bound (7.5e-5, plus float32 rounding)
    against torch's float32 exp2, over the softmax's argument range."""
    x = torch.linspace(-100.0, 8.0, 1_000_001, device="cuda", dtype=torch.float32)
    y = lc.debug_exp2_poly(x)
    ref = torch.exp2(x.double())
    rel = ((y.double() - ref).abs() / ref).max().item()
    assert rel < 1.0e-4
    # far below the range it returns (almost) zero, never garbage
    z = lc.debug_exp2_poly(torch.tensor([-float("inf"), -1e30, -300.0, -127.0, -126.4], device="cuda"))
    assert torch.isfinite(z).all() and (z >= 0).all() and (z < 1e-37).all()


def test_wide_logit_range(lc):
    """Q scaled by 30: logits spread over hundreds of log2 units, so the
    exponentials see arguments far below the polynomial's clamp and the lazy
    rescale of O triggers; the output still matches the oracle."""
    w = li.Workload("wide", B=1, H=2, D=128, Y=16, X=24, q_frames=2, kv_past=(4,), cap_frames=6,
                    density=0.5, seed=61)
    x = li.make_inputs(w)
    x["q"] = (x["q"].float() * 30.0).to(torch.bfloat16)
    g = run_gpu(lc, w, x)
    assert g["err"] == 0
    assert np.isfinite(g["O"]).all()
    compare_all(w, x, g)
