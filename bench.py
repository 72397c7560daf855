"""Benchmark: one streaming LCSA step per 8-frame chunk at 768x1408 on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload chunk|multistream|uhr_truncate|uhr_preserve|uhr_truncate_tok|
                                uhr_preserve_tok|clip|clip_5|clip_30]
                    [--mode fwd|bwd|segment]

A step is the whole hot path over one chunk: lcsa_pool_qk (Q), lcsa_kv_append
(K, V and K pooled on the way into the ring cache, evicting the oldest frames),
lcsa_select_blocks (coarse map, causal mask, top-K) and lcsa_sparse_attn_fwd,
with Q/K/V resident in HBM. L2 is flushed (a 512 MB write and a 256 MB read)
before every timed step, outside the timed events. The step is timed twice:
eagerly with CUDA events between the kernels (the per-kernel split) and
replayed from a CUDA graph (the headline value: the same kernels and work,
one launch). Under torchrun each rank streams its own independent video (weak
scaling, no data-path collective); the step time is the max over ranks.

--mode bwd times the attention backward on a whole clip (training form);
--mode segment the stage-1 dense segment attention, forward and backward.

Rank 0 prints one JSON line. `--impl reference` times the fp64 CPU oracle on
a bounded sample of the same workload instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

import lcsa_inputs as li  # noqa: E402

METRIC = "ms per 8-frame chunk at 768x1408; sparse-attn TFLOP/s and % of BF16/HBM roofline"
UNIT = "ms/chunk"
CHUNKS_PER_STEP = {"clip": 13, "clip_5": 13, "clip_30": 13}  # a whole clip is 13 two-frame chunks

WORKLOAD_TEXT = {
    "chunk": "768x1408 streaming chunk: 12 heads, d=128, 48x88 tokens/frame, 2-frame query chunk "
             "vs 6-frame KV cache (chunk + 4 past), 3D RoPE, 13.6% of causal block pairs",
    "multistream": "4 streams at 768x1408, 2-frame chunks, ragged 4/5/6 past frames, 13.6%",
    "uhr_truncate": "1536x2688: 96x168 tokens/frame, 2+4 frames, 9x9-block window, truncate, 13.6%",
    "uhr_preserve": "1536x2688: 96x168 tokens/frame, 2+4 frames, 9x9-block window, preserve, 13.6%",
    "uhr_truncate_tok": "1536x2688: 96x168 tokens/frame, 2+4 frames, 72x72-token window per query token, "
                        "truncate, 13.6%",
    "uhr_preserve_tok": "1536x2688: 96x168 tokens/frame, 2+4 frames, 72x72-token window per query token, "
                        "preserve, 13.6%",
    "clip": "whole 101-frame clip at 768x1408: 26 latent frames, block-causal, 13.6%",
    "clip_5": "whole 101-frame clip at 768x1408: 26 latent frames, block-causal, 5%",
    "clip_30": "whole 101-frame clip at 768x1408: 26 latent frames, block-causal, 30%",
}


ATTN_SOURCES = ("block_sparse_causal_lcsa_b200/csrc/attn_fwd.cuh",
                "block_sparse_causal_lcsa_b200/csrc/lcsa_device.cuh")


def attn_source_hash() -> str:
    """Hash of the attention kernel's sources: DRAM traffic captured by ncu is
    reported only while the kernel is unchanged since the capture."""
    import hashlib
    h = hashlib.sha256()
    for f in ATTN_SOURCES:
        h.update(open(os.path.join(ROOT, f), "rb").read())
    return h.hexdigest()[:16]


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained"), "sm_max_mhz": d.get("sm_max_mhz"),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


class ClockSampler:
    """nvidia-smi clock / throttle sampling while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            import tempfile
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            parts = [s.strip() for s in line.split(",")]
            if len(parts) >= 9:
                rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        smax = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None, "reasons": reasons,
                "samples": len(rows)}


def dist_setup(n_gpus: int):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int, device="cuda") -> float:
    """The largest of the ranks' values (every rank gets it). The only
    collective besides the barrier: the data path exchanges nothing."""
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_workload(w: "li.Workload", rank: int) -> "li.Workload":
    """Rank r streams its own video: the same shapes, seed + 1000 r (weak scaling)."""
    return li.Workload(**{**w.__dict__, "seed": w.seed + 1000 * rank})


def whole_job_ms_per_chunk(step_ms_max: float, chunks_per_rank_step: int, world: int) -> float:
    """All ranks process their chunks side by side in the slowest rank's step time."""
    return step_ms_max / (chunks_per_rank_step * world)


def attn_flops(blk_cnt: torch.Tensor, blk_idx: torch.Tensor, cache, Hb: int, Wb: int, D: int,
               q_tokens_per_block: int = 128) -> float:
    """4*D*sum(q tokens x kept key tokens); a one-frame key block counts 64 keys."""
    cnt = blk_cnt.long().cpu()
    idx = blk_idx.long().cpu()
    total = 0
    for b in range(cnt.shape[0]):
        keys = cnt[b].sum().item() * 128
        if cache.begin(b) % 2 == 1:  # oldest cached block has one frame
            valid = torch.arange(idx.shape[-1]).view(1, 1, -1) < cnt[b].unsqueeze(-1)
            n_partial = ((idx[b] < Hb * Wb) & (idx[b] >= 0) & valid).sum().item()
            keys -= 64 * n_partial
        total += keys
    return 4.0 * D * q_tokens_per_block * total


# ----------------------------------------------------------------------------- our arm
def make_flusher(dev):
    """L2 flush: write 512 MB, then read another 256 MB so that the written
    (dirty) lines are written back before the next timed region starts."""
    flush = torch.empty(512 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
    flush_rd = torch.ones(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)

    def flush_l2():
        flush.zero_()
        flush_rd.sum()
    return flush_l2


def allowed_pairs(w, cache) -> int:
    """Number of (query block, key block) pairs the coarse map scores: causal
    candidates inside the query block's window (all of them without one)."""
    nQT = (w.q_frames + 1) // 2

    def axis_sizes(n):
        out = []
        for i in range(n):
            if w.window <= 0:
                lo, hi = 0, n
            elif w.window_mode >= 2:      # token windows: blocks seen by some token of block i
                def tw(t, ntok):
                    s0 = t - w.window // 2
                    if w.window_mode == 2:
                        return max(s0, 0), min(s0 + w.window, ntok)
                    st = max(min(s0, ntok - w.window), 0)
                    return st, min(st + w.window, ntok)
                a, _ = tw(8 * i, 8 * n)
                _, d = tw(8 * i + 7, 8 * n)
                lo, hi = a // 8, (d - 1) // 8 + 1
            elif w.window_mode == 0:
                r = w.window // 2
                lo, hi = max(i - r, 0), min(i + r + 1, n)
            else:
                r = w.window // 2
                lo = max(min(i - r, n - w.window), 0)
                hi = min(lo + w.window, n)
            out.append(hi - lo)
        return out
    area = sum(a * b for a in axis_sizes(w.Hb) for b in axis_sizes(w.Wb))
    total = 0
    for b in range(w.B):
        nKT = cache.end(b) // 2 - cache.begin(b) // 2
        for tq in range(nQT):
            total += (nKT - nQT + tq + 1) * area
    return total * w.H


def setup_workload(lc, w, x, dev, n_chunks=3):
    """Device state of one workload and the functions that run one step of it.

    Streaming workloads: a ring cache holding each stream's past frames, then
    per step lcsa_ingest_chunk (Q pooled, K pooled while K and V are written
    into the ring), lcsa_select_blocks and lcsa_sparse_attn_fwd, on distinct
    chunks cycled through the steps. Whole clip: Q, K, V of all 26 frames
    resident, per step lcsa_pool_qk (Q and K), select and attention."""
    params = lc.SelectParams(top_k=w.top_k, density=w.density, window=w.window, window_mode=w.window_mode)
    st = type("Setup", (), {})()
    st.w = w
    st.streaming = w.kv_past[0] > 0 or w.B > 1
    tok_window = w.window if w.window_mode >= li.WINDOW_TRUNCATE_TOKENS else 0
    if st.streaming:
        cache = lc.KVCache(w.B, w.H, w.cap_frames, w.Y, w.X, w.D, device=dev)
        for b in range(w.B):
            kp = x["k"][b][:, :w.kv_past[b]].unsqueeze(0).to(dev)
            vp = x["v"][b][:, :w.kv_past[b]].unsqueeze(0).to(dev)
            lc.kv_append(cache, kp, vp, lc.pool_qk(kp)[0], stream_offset=b)
        g = torch.Generator().manual_seed(w.seed + 7)
        shp = (w.B, w.H, w.q_frames, w.Y, w.X, w.D)
        chunks = [(x["q"].to(dev),
                   torch.stack([x["k"][b][:, -w.q_frames:] for b in range(w.B)]).to(dev),
                   torch.stack([x["v"][b][:, -w.q_frames:] for b in range(w.B)]).to(dev))]
        for _ in range(n_chunks - 1):
            chunks.append(tuple(torch.randn(shp, generator=g).to(torch.bfloat16).to(dev) for _ in range(3)))
        step = lc.StreamingStep(cache, w.q_frames, params)
        base_state = cache.state()

        def run_step(i, ev=None):
            q, k, v = chunks[i % n_chunks]
            # every step sees the workload's cache lengths (host-side state only);
            # the append still writes the chunk's frames and pooled K into the ring
            step.cache.set_state(base_state)
            if ev is not None:
                ev[0].record()
            lc.ingest_chunk(q, step.cache, k, v, step.q_pool)
            if ev is not None:
                ev[1].record()
            lc.select_blocks(step.q_pool, step.q_frames, step.cache, step.params, step.kmax,
                             step.blk_idx, step.blk_cnt, step.workspace)
            if ev is not None:
                ev[2].record()
            lc.sparse_attn_fwd(q, step.cache, step.blk_idx, step.blk_cnt, step.o, step.lse,
                               workspace=step.attn_ws, window=tok_window, window_mode=w.window_mode)
            if ev is not None:
                ev[3].record()
            return step.o

        def run_split(i, ev):
            # the ingest as two launches: Q pooling alone, then the K/V append
            q, k, v = chunks[i % n_chunks]
            step.cache.set_state(base_state)
            ev[0].record()
            lc.pool_qk(q, None, step.q_pool)
            ev[1].record()
            lc.kv_append(step.cache, k, v)
            ev[2].record()

        def graph_step():
            step.cache.set_state(base_state)
            step.graph_step()

        st.kernels = ["ingest", "select", "attn"]
        st.split_kernels = ["pool", "kv_append"]
        st.run_split = run_split
        st.graph_prepare = lambda: (step.cache.set_state(base_state), step.graph_step(*chunks[0]))
        st.graph_step = graph_step
        st.cache, st.step, st.chunks, st.base_state = cache, step, chunks, base_state
        st.blk_idx, st.blk_cnt, st.o = step.blk_idx, step.blk_cnt, step.o
        st.kmax = step.kmax
    else:
        q = x["q"].to(dev)
        k = x["k"][0].unsqueeze(0).to(dev)
        v = x["v"][0].unsqueeze(0).to(dev)
        q_pool = torch.empty(lc.api.pooled_shape(q), dtype=torch.float64, device=dev)
        k_pool = torch.empty(lc.api.pooled_shape(k), dtype=torch.float64, device=dev)
        cache = lc.KVCache.wrap(k, v, k_pool)
        kmax = lc.select_kmax(cache, w.q_frames, params)
        nQB = q_pool.shape[2] * q_pool.shape[3] * q_pool.shape[4]
        blk_idx = torch.empty((1, w.H, nQB, kmax), dtype=torch.int32, device=dev)
        blk_cnt = torch.empty((1, w.H, nQB), dtype=torch.int32, device=dev)
        o = torch.empty_like(q)
        lse = torch.empty(q.shape[:5], dtype=torch.float32, device=dev)
        sel_ws = torch.empty(max(lc.select_workspace_bytes(cache, w.q_frames), 16), dtype=torch.uint8, device=dev)
        attn_ws = lc.attn_workspace(w.D, dev)

        def run_step(i, ev=None):
            if ev is not None:
                ev[0].record()
            lc.pool_qk(q, k, q_pool, k_pool)
            if ev is not None:
                ev[1].record()
            lc.select_blocks(q_pool, w.q_frames, cache, params, kmax, blk_idx, blk_cnt, sel_ws)
            if ev is not None:
                ev[2].record()
            lc.sparse_attn_fwd(q, cache, blk_idx, blk_cnt, o, lse, workspace=attn_ws)
            if ev is not None:
                ev[3].record()
            return o

        st.kernels = ["pool", "select", "attn"]
        st.split_kernels = []
        st.graph_step = None
        st.cache, st.q, st.k, st.v = cache, q, k, v
        st.blk_idx, st.blk_cnt, st.o = blk_idx, blk_cnt, o
        st.kmax = kmax
    st.run_step = run_step
    return st


def time_events(n, nev, body, flush_l2):
    """n timed repetitions of body(i, ev) with L2 flushed before each (outside
    the events); returns the per-repetition lists of event-pair durations."""
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(nev)] for _ in range(n)]
    for i in range(n):
        flush_l2()
        body(i, evs[i])
    torch.cuda.synchronize()
    return [[evs[i][j].elapsed_time(evs[i][j + 1]) for j in range(nev - 1)] for i in range(n)]


def measure(lc, st, steps, warmup, flush_l2, peaks, world, clocks=None):
    """Per-kernel split (eager, CUDA events between the kernels), the
    whole-step graph replay, and the derived rooflines of one workload."""
    w = st.w
    for i in range(warmup):
        flush_l2()
        st.run_step(i)
    torch.cuda.synchronize()
    if lc.last_device_error() != 0:
        raise RuntimeError("device error during warm-up (%s)" % w.name)
    barrier(world)
    torch.cuda.synchronize()
    if clocks is not None:
        clocks.start()
        time.sleep(0.3)
    t_wall = time.perf_counter()
    eager = time_events(steps, len(st.kernels) + 1, lambda i, ev: st.run_step(warmup + i, ev), flush_l2)
    split = (time_events(steps, len(st.split_kernels) + 1, st.run_split, flush_l2)
             if st.split_kernels else None)
    graph_ms = None
    if st.graph_step is not None:
        st.graph_prepare()
        for _ in range(warmup):
            flush_l2()
            st.graph_step()
        g = time_events(steps, 2, lambda i, ev: (ev[0].record(), st.graph_step(), ev[1].record()), flush_l2)
        graph_ms = statistics.mean(r[0] for r in g)
    torch.cuda.synchronize()
    t_wall = time.perf_counter() - t_wall
    barrier(world)
    clk = None
    if clocks is not None:
        time.sleep(0.2)
        clk = clocks.stop()
    if lc.last_device_error() != 0:
        raise RuntimeError("device error during the timed steps (%s)" % w.name)

    per_kernel = {k: statistics.mean(r[j] for r in eager) for j, k in enumerate(st.kernels)}
    if split is not None:
        per_kernel.update({k: statistics.mean(r[j] for r in split) for j, k in enumerate(st.split_kernels)})
    eager_ms = max_over_ranks(statistics.mean(sum(r) for r in eager), world)
    chunks_per_step = CHUNKS_PER_STEP.get(w.name, 1) * w.B
    res = {"eager_ms_per_chunk": whole_job_ms_per_chunk(eager_ms, chunks_per_step, world),
           "graph_ms_per_chunk": (whole_job_ms_per_chunk(max_over_ranks(graph_ms, world), chunks_per_step, world)
                                  if graph_ms is not None else None),
           "per_kernel_ms": per_kernel, "clocks": clk, "wall_s_timed": t_wall}

    # attention: algorithmic FLOPs of the kept blocks, tensor-bound
    flops = attn_flops(st.blk_cnt, st.blk_idx, st.cache, w.Hb, w.Wb, w.D)
    tflops = flops / (per_kernel["attn"] / 1e3) / 1e12
    res["attn"] = {"flops": flops, "tflops": tflops, "frac": tflops / peaks["bf16_tflops"]}

    # HBM-side launches: algorithmic bytes per launch
    tokens_q = w.B * w.H * w.q_frames * w.Y * w.X
    pooled_row = w.D * 8
    hbm = {}
    if st.streaming:
        tokens_kv = tokens_q                                  # the chunk's new K / V frames
        bytes_pool = tokens_q * w.D * 2 + (tokens_q // 128) * pooled_row
        bytes_app = 2 * (2 * tokens_kv * w.D * 2) + (tokens_kv // 128) * pooled_row
        hbm["pool_gbs"] = bytes_pool / (per_kernel["pool"] / 1e3) / 1e9
        hbm["kv_append_gbs"] = bytes_app / (per_kernel["kv_append"] / 1e3) / 1e9
        hbm["ingest_gbs"] = (bytes_pool + bytes_app) / (per_kernel["ingest"] / 1e3) / 1e9
        res["bytes"] = {"pool": bytes_pool, "kv_append": bytes_app, "ingest": bytes_pool + bytes_app}
    else:
        bytes_pool = 2 * tokens_q * w.D * 2 + 2 * (tokens_q // 128) * pooled_row
        hbm["pool_gbs"] = bytes_pool / (per_kernel["pool"] / 1e3) / 1e9
        res["bytes"] = {"pool": bytes_pool}
    res["hbm"] = {k: v / peaks["hbm_gbs"] for k, v in hbm.items()}
    res["hbm_gbs"] = hbm

    # selection: bytes it must move (pooled Q and the candidates' pooled K in,
    # block lists out) and its float64 work (one multiply and one add per
    # channel of every scored pair)
    rows = w.B * w.H * ((w.q_frames + 1) // 2) * w.Hb * w.Wb
    n_kblocks = sum((st.cache.end(b) // 2 - st.cache.begin(b) // 2) for b in range(w.B)) * w.Hb * w.Wb * w.H
    sel_bytes = rows * pooled_row + n_kblocks * pooled_row + rows * st.kmax * 4 + rows * 4
    pairs = allowed_pairs(w, st.cache)
    sel_s = per_kernel["select"] / 1e3
    fp64_tflops = 2.0 * w.D * pairs / sel_s / 1e12
    q_pool_bytes = rows * pooled_row + (tokens_q * w.D * 2)            # the Q pooling launch
    pool_ms = per_kernel["pool"]
    res["select"] = {
        "ms": per_kernel["select"], "bytes": sel_bytes, "gbs": sel_bytes / sel_s / 1e9,
        "hbm_frac": sel_bytes / sel_s / 1e9 / peaks["hbm_gbs"],
        "scored_pairs": pairs, "fp64_tflops": fp64_tflops, "fp64_frac": fp64_tflops / FP64_PEAK_TFLOPS,
        "pool_plus_select_gbs": (q_pool_bytes + sel_bytes) / ((pool_ms + per_kernel["select"]) / 1e3) / 1e9,
    }
    res["select"]["pool_plus_select_hbm_frac"] = res["select"]["pool_plus_select_gbs"] / peaks["hbm_gbs"]
    return res


# float64 peak for the selection's roofline: 148 SMs x 64 FP64 lanes x 2 FLOP
# (a fused multiply-add) x 1965 MHz (the B200's maximum SM clock); the score
# kernel issues a separate multiply and add per channel, so its instruction
# peak is the same 18.6 T instructions/s counted as 2 FLOP each.
FP64_PEAK_TFLOPS = 148 * 64 * 2 * 1.965e9 / 1e12


EXTRA_WORKLOADS = ["multistream", "uhr_truncate", "uhr_preserve", "uhr_truncate_tok", "uhr_preserve_tok",
                   "clip_5", "clip", "clip_30"]


def run_ours(args, world, rank, local):
    import block_sparse_causal_lcsa_b200 as lc

    dev = torch.device("cuda", local)
    peaks = load_peaks()
    # each rank streams an independent video (weak scaling)
    w = rank_workload(li.workload(args.workload), rank)
    x = li.make_inputs(w)
    st = setup_workload(lc, w, x, dev)
    flush_l2 = make_flusher(dev)
    clocks = ClockSampler(local)
    m = measure(lc, st, args.steps, args.warmup, flush_l2, peaks, world, clocks=clocks)
    chunks_per_step = CHUNKS_PER_STEP.get(args.workload, 1) * w.B
    per_kernel = m["per_kernel_ms"]

    # e2e: the same step through the API with the chunk's inputs coming from
    # pinned host memory and O going back there, copies inside the timed region
    e2e = None
    if st.streaming:
        # distinct pinned host chunks through the library's own pipeline
        # (lcsa_pipeline_*: the C ABI takes the host buffers): each chunk's
        # inputs cross PCIe while the previous chunk computes, and its O comes
        # back on a third stream; the timed region runs, on the pipeline's own
        # events, from the first timed chunk's host-to-device copy to the last
        # chunk's device-to-host copy. No L2 flush in this loop: every step's
        # inputs arrive by a fresh copy and its working set (cache + chunk) is
        # larger than L2.
        host = [tuple(t.cpu().pin_memory() for t in c) for c in st.chunks]
        ho = torch.empty(host[0][0].shape, dtype=torch.bfloat16).pin_memory()
        pipe = lc.NativePipeline(st.step.cache, w.q_frames, st.step.params)
        for i in range(args.warmup + args.steps):
            if i == args.warmup:
                pipe.sync()
                pipe.start_timer()
            st.step.cache.set_state(st.base_state)
            pipe.submit(*host[i % len(host)], ho)
        pipe.sync()
        e2e_ms = max_over_ranks(pipe.elapsed_ms() / args.steps, world)
        pipe.close()
        st.step.cache.set_state(st.base_state)
        hq, hk, hv = host[0]
        e2e = {"value": whole_job_ms_per_chunk(e2e_ms, chunks_per_step, world), "unit": UNIT,
               "h2d_bytes_per_step": hq.numel() * 2 + hk.numel() * 2 + hv.numel() * 2,
               "d2h_bytes_per_step": ho.numel() * 2,
               "api": "lcsa_pipeline_submit (C ABI, host buffers)",
               "pipelined": "copies of chunk i+1 overlap the compute of chunk i; "
                            "%d distinct host chunks cycled; no L2 flush (inputs arrive by copy)" % len(host)}
    else:
        hq, hk, hv = st.q.cpu().pin_memory(), st.k.cpu().pin_memory(), st.v.cpu().pin_memory()
        ho = torch.empty(hq.shape, dtype=torch.bfloat16).pin_memory()
        e_start = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
        e_end = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
        for i in range(args.warmup + args.steps):
            if i >= args.warmup:
                e_start[i - args.warmup].record()
            st.q.copy_(hq, non_blocking=True)
            st.k.copy_(hk, non_blocking=True)
            st.v.copy_(hv, non_blocking=True)
            out = st.run_step(i)
            ho.copy_(out, non_blocking=True)
            if i >= args.warmup:
                e_end[i - args.warmup].record()
        torch.cuda.synchronize()
        e2e_ms = max_over_ranks(statistics.mean(a.elapsed_time(b) for a, b in zip(e_start, e_end)), world)
        e2e = {"value": whole_job_ms_per_chunk(e2e_ms, chunks_per_step, world), "unit": UNIT,
               "h2d_bytes_per_step": (hq.numel() + hk.numel() + hv.numel()) * 2,
               "d2h_bytes_per_step": ho.numel() * 2}
    if lc.last_device_error() != 0:
        raise RuntimeError("device error during the end-to-end steps")

    traffic = None
    tfile = os.path.join(ROOT, "profiles", "attn_fwd_%s.traffic.txt" % args.workload)
    if os.path.exists(tfile):
        rec = dict(line.split(":", 1) for line in open(tfile) if ":" in line and not line.startswith("#"))
        if rec.get("source_hash", "").strip() == attn_source_hash():
            traffic = int(rec["bytes_per_launch"])

    # kernels per timed step of the headline (graph replay): the ingest
    # (streaming: one fused launch; clip: Q and K pooling), score + top-K, the
    # attention and, when its last wave is split, the merge of the halves
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    units = w.B * w.H * ((w.q_frames + 1) // 2) * w.Hb * w.Wb
    split = units > sms and 0 < units % sms <= sms // 2
    launches_per_step = 1 + 2 + (2 if split else 1)
    # the headline is the step as a user runs it in production: replayed from a
    # CUDA graph (same kernels, same work, one launch); the eager run with CUDA
    # events between the kernels gives the per-kernel split
    value = m["graph_ms_per_chunk"] if m["graph_ms_per_chunk"] is not None else m["eager_ms_per_chunk"]
    step_ms = value * chunks_per_step * world
    peak = peaks["bf16_tflops"]
    clk = m["clocks"]
    sm_mhz = (clk or {}).get("sm_mhz") or peaks.get("sm_max_mhz") or 1965.0
    line = {
        "metric": METRIC, "value": round(value, 4), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(step_ms, 4),
        "eager_ms_per_chunk": round(m["eager_ms_per_chunk"], 4),
        "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) bf16, shapes of the pages' 768x1408 workload)",
        "config": {"workload": WORKLOAD_TEXT[args.workload], "name": args.workload,
                   "streams_per_gpu": w.B, "heads": w.H, "head_dim": w.D,
                   "tokens_per_frame": w.Y * w.X, "q_frames": w.q_frames,
                   "kv_frames": list(w.kv_frames), "density": w.density, "window": w.window,
                   "l2": "flushed before every timed step (512 MB write, then 256 MB read)",
                   "select_precision": "fp64 scores, exact top-K",
                   "parallelism": "independent stream per GPU" if world > 1 else "single GPU"},
        "per_kernel_ms": {k2: round(v2, 5) for k2, v2 in per_kernel.items()},
        "sparse_attn_tflops": round(m["attn"]["tflops"], 2),
        "roofline": {"bound": "tensor", "kernel": "attn_fwd", "achieved": round(m["attn"]["tflops"], 2),
                     "peak": peak, "unit": "TFLOP/s", "frac": round(m["attn"]["tflops"] / peak, 4),
                     "peak_source": "%s bf16 burst (MEASURED_PEAKS.json)" % peaks["source"],
                     "flops_per_launch": m["attn"]["flops"], "traffic": traffic,
                     # the same FLOPs against the dense bf16 tensor peak at the SM clock
                     # sampled during the run (8192 FLOP per clock per SM x 148 SMs)
                     "frac_of_clock_peak": round(m["attn"]["tflops"] / (148 * 8192 * sm_mhz * 1e6 / 1e12), 4),
                     "clock_peak_tflops": round(148 * 8192 * sm_mhz * 1e6 / 1e12, 1)},
        "hbm_kernels": {k2: round(v2, 1) for k2, v2 in m["hbm_gbs"].items()},
        "hbm_frac": {k2: round(v2, 4) for k2, v2 in m["hbm"].items()},
        "select": {k2: (round(v2, 5) if isinstance(v2, float) else v2) for k2, v2 in m["select"].items()},
        "select_fp64_peak": "%.1f TFLOP/s = 148 SMs x 64 FP64 lanes x 2 FLOP x 1965 MHz (nominal)" % FP64_PEAK_TFLOPS,
        "cuda_graph": ({"ms_per_chunk": round(m["graph_ms_per_chunk"], 4), "graph_launches_per_step": 1}
                       if m["graph_ms_per_chunk"] is not None else None),
        "hbm_peak_gbs": peaks["hbm_gbs"],
        "e2e": e2e,
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clk,
        "wall_s_timed": round(m["wall_s_timed"], 4),
    }
    del st
    torch.cuda.empty_cache()
    if not args.no_workloads and world == 1:
        line["workloads"] = extra_workloads(lc, dev, peaks, args, flush_l2)
    if rank == 0 and not args.no_cpu_baseline and world == 1:
        line["cpu_baseline"] = cpu_baseline(w, x, budget_s=args.cpu_budget)
    return line


def extra_workloads(lc, dev, peaks, args, flush_l2):
    """The other configurations of the metric, a few steps each: ms per chunk
    (graph replay for streams, eager for the whole clip, divided by its 13
    chunks), attention TFLOP/s and fraction of the bf16 peak, selection."""
    out = {}
    cache_inputs = {}
    for name in EXTRA_WORKLOADS:
        w = li.workload(name)
        key = (w.seed, w.structure, w.B, w.Y, w.X, w.q_frames, w.kv_past)
        if key not in cache_inputs:
            cache_inputs.clear()
            cache_inputs[key] = li.make_inputs(w)
        x = cache_inputs[key]
        st = setup_workload(lc, w, x, dev)
        m = measure(lc, st, args.extra_steps, 3, flush_l2, peaks, 1)
        out[name] = {
            "ms_per_chunk": round(m["graph_ms_per_chunk"] if m["graph_ms_per_chunk"] is not None
                                  else m["eager_ms_per_chunk"], 4),
            "timed_as": "graph replay" if m["graph_ms_per_chunk"] is not None else "eager, clip / 13 chunks",
            "attn_ms": round(m["per_kernel_ms"]["attn"], 4),
            "attn_tflops": round(m["attn"]["tflops"], 1), "attn_frac": round(m["attn"]["frac"], 4),
            "select_ms": round(m["select"]["ms"], 4), "select_fp64_frac": round(m["select"]["fp64_frac"], 4),
            "pool_gbs": round(m["hbm_gbs"]["pool_gbs"], 1),
            "ingest_gbs": round(m["hbm_gbs"].get("ingest_gbs", float("nan")), 1) if st.streaming else None,
            "kept_pairs": int(st.blk_cnt.sum().item()),
        }
        del st, m
        torch.cuda.empty_cache()
    return out


# ----------------------------------------------------------------------------- oracle arm
def backward_cpu_baseline(w, x, d_o, budget_s):
    """The oracle's attention backward as it stands, timed on host cores on a
    bounded sample: the oracle selects the blocks of head 0 of stream 0 itself,
    then attend_rows_backward runs on its query blocks in order until the
    budget is spent. Scaled by kept block pairs to the whole workload: K_i
    depends only on the geometry (causality, window, density), so every head
    of a stream keeps as many pairs as its head 0."""
    from oracle import lcsa_oracle as orc

    qh, kh, vh = orc.widen(x["q"][0, 0]), orc.widen(x["k"][0][0]), orc.widen(x["v"][0][0])
    Tq, Y, X, D = qh.shape
    sel, total_kept = None, 0
    for b in range(w.B):
        qb = qh if b == 0 else orc.widen(x["q"][b, 0])
        kb = kh if b == 0 else orc.widen(x["k"][b][0])
        sb, Ks, _ = orc.select_head(orc.pool_blocks(qb), orc.pool_blocks(kb), Tq, kb.shape[0], Y, X,
                                    w.top_k, w.density, w.window, w.window_mode)
        total_kept += int(Ks.sum()) * w.H
        if b == 0:
            sel = sb
    q2, k2, v2 = qh.reshape(-1, D), kh.reshape(-1, D), vh.reshape(-1, D)
    g2 = orc.widen(d_o[0, 0]).reshape(-1, D)
    n_rows = kept = 0
    with CpuMeter() as meter:
        for i in range(len(sel)):
            qidx = orc.block_token_index(Tq, Y, X, [i])
            kidx = orc.block_token_index(kh.shape[0], Y, X, sel[i])
            orc.attend_rows_backward(q2[qidx], k2[kidx], v2[kidx], g2[qidx])
            n_rows += 1
            kept += len(sel[i])
            if time.perf_counter() - meter.w0 > budget_s:
                break
    return {"value": round(meter.wall / kept * total_kept * 1e3, 1), "unit": "ms/clip", "cores": meter.cores,
            "cpu_model": cpu_model(), "kind": "oracle", "kept_pairs_total": total_kept,
            "sample": "%d query blocks (%d kept block pairs) of head 0, blocks selected by the oracle, "
                      "attend_rows_backward in fp64, scaled by kept pairs to all %d" % (n_rows, kept, total_kept)}


def run_backward(args, world, rank, local):
    """Attention gradients for training with the block-sparse causal mask: the
    whole clip is the key timeline, the forward runs once (untimed), then each
    step is one lcsa_sparse_attn_bwd call (prep, transposed lists, dQ, dK/dV)."""
    import block_sparse_causal_lcsa_b200 as lc

    w = rank_workload(li.workload(args.workload), rank)
    dev = torch.device("cuda", local)
    peaks = load_peaks()
    x = li.make_inputs(w)
    cache = lc.KVCache(w.B, w.H, w.cap_frames, w.Y, w.X, w.D, device=dev)
    for b in range(w.B):
        kb = x["k"][b].unsqueeze(0).to(dev)
        vb = x["v"][b].unsqueeze(0).to(dev)
        lc.kv_append(cache, kb, vb, stream_offset=b)
    q = x["q"].to(dev)
    params = lc.SelectParams(top_k=w.top_k, density=w.density, window=w.window, window_mode=w.window_mode)
    idx, cnt = lc.select_blocks(lc.pool_qk(q)[0], w.q_frames, cache, params)
    o, lse = lc.sparse_attn_fwd(q, cache, idx, cnt)
    g = torch.Generator().manual_seed(w.seed + 11)
    d_o_host = torch.randn(q.shape, generator=g).to(torch.bfloat16)
    d_o = d_o_host.to(dev)
    dq, dk, dv = torch.empty_like(q), torch.zeros_like(cache.k), torch.zeros_like(cache.v)
    ws = torch.empty(max(lc.sparse_attn_bwd_workspace_bytes(cache, w.q_frames), 16), dtype=torch.uint8, device=dev)
    flush = torch.empty(512 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)

    def step():
        lc.sparse_attn_bwd(q, cache, idx, cnt, o, lse, d_o, dq, dk, dv, ws)

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    if lc.last_device_error() != 0:
        raise RuntimeError("device error during warm-up")
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    clocks = ClockSampler(local)
    barrier(world)
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.3)
    for a, b in evs:
        flush.zero_()
        a.record()
        step()
        b.record()
    torch.cuda.synchronize()
    barrier(world)
    time.sleep(0.2)
    clk = clocks.stop()
    if lc.last_device_error() != 0:
        raise RuntimeError("device error during the timed steps")
    ms = max_over_ranks(statistics.mean(a.elapsed_time(b) for a, b in evs), world)
    fwd_flops = attn_flops(cnt, idx, cache, w.Hb, w.Wb, w.D)
    algo_flops = 2.5 * fwd_flops        # dS/dP, dQ, dK, dV and the recomputed S: 5 products
    exec_flops = 3.5 * fwd_flops        # this implementation: S and dP in both kernels, 7 products
    achieved = algo_flops / (ms / 1e3) / 1e12
    line = {
        "metric": "ms per attention backward of a 101-frame 768x1408 clip (training, block-sparse causal)",
        "value": round(ms / world, 4), "unit": "ms/clip", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms, 4), "higher_is_better": False, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded, shapes of the pages' clip workload)",
        "config": {"workload": WORKLOAD_TEXT[args.workload], "name": args.workload, "mode": "backward",
                   "l2": "flushed before every timed step (512 MB write)"},
        "roofline": {"bound": "tensor", "kernel": "attention backward (4 launches)", "achieved": round(achieved, 2),
                     "peak": peaks["bf16_tflops"], "unit": "TFLOP/s", "frac": round(achieved / peaks["bf16_tflops"], 4),
                     "peak_source": "measured bf16 burst (MEASURED_PEAKS.json)" if peaks["source"] == "measured"
                     else "fallback", "flops_algorithmic": algo_flops, "flops_executed": exec_flops,
                     "executed_tflops": round(exec_flops / (ms / 1e3) / 1e12, 2), "traffic": None},
        "gpu_launches": 4 * args.steps,
        "clocks": clk,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = backward_cpu_baseline(w, x, d_o_host, args.cpu_budget)
    return line


def run_segment(args, world, rank, local):
    """Stage-1 dense attention confined to segments (video clips and images):
    segment block lists, then the attention forward and backward; each step is
    one forward and one backward of the batch (the block lists are built once)."""
    import block_sparse_causal_lcsa_b200 as lc

    w = li.SEGMENT_WORKLOADS["joint"]
    w = li.SegmentWorkload(**{**w.__dict__, "seed": w.seed + 1000 * rank})
    dev = torch.device("cuda", local)
    peaks = load_peaks()
    x = li.make_segment_inputs(w)
    cache = lc.KVCache(w.B, w.H, w.cap_frames, w.Y, w.X, w.D, device=dev)
    for b in range(w.B):
        lc.kv_append(cache, x["k"][b].unsqueeze(0).to(dev), x["v"][b].unsqueeze(0).to(dev), stream_offset=b)
    q = x["q"].to(dev)
    idx, cnt = lc.segment_blocks(w.q_frames, cache)
    o = torch.empty_like(q)
    lse = torch.empty(q.shape[:5], dtype=torch.float32, device=dev)
    g = torch.Generator().manual_seed(w.seed + 11)
    d_o = torch.randn(q.shape, generator=g).to(torch.bfloat16)
    for b, F in enumerate(w.seg_frames):
        d_o[b, :, :w.q_frames - F] = 0
    d_o = d_o.to(dev)
    dq, dk, dv = torch.empty_like(q), torch.zeros_like(cache.k), torch.zeros_like(cache.v)
    ws = torch.empty(max(lc.sparse_attn_bwd_workspace_bytes(cache, w.q_frames), 16), dtype=torch.uint8, device=dev)
    flush = torch.empty(512 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)

    def step(ev=None):
        if ev is not None:
            ev[0].record()
        lc.sparse_attn_fwd(q, cache, idx, cnt, o, lse)
        if ev is not None:
            ev[1].record()
        lc.sparse_attn_bwd(q, cache, idx, cnt, o, lse, d_o, dq, dk, dv, ws)
        if ev is not None:
            ev[2].record()

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    if lc.last_device_error() != 0:
        raise RuntimeError("device error during warm-up")
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    clocks = ClockSampler(local)
    barrier(world)
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.3)
    for ev in evs:
        flush.zero_()
        step(ev)
    torch.cuda.synchronize()
    barrier(world)
    time.sleep(0.2)
    clk = clocks.stop()
    if lc.last_device_error() != 0:
        raise RuntimeError("device error during the timed steps")
    fwd_ms = max_over_ranks(statistics.mean(e[0].elapsed_time(e[1]) for e in evs), world)
    bwd_ms = max_over_ranks(statistics.mean(e[1].elapsed_time(e[2]) for e in evs), world)
    fwd_flops = attn_flops(cnt, idx, cache, w.Y // 8, w.X // 8, w.D)
    f_tf = fwd_flops / (fwd_ms / 1e3) / 1e12
    b_tf = 2.5 * fwd_flops / (bwd_ms / 1e3) / 1e12
    peak = peaks["bf16_tflops"]
    return {
        "metric": "ms per attention forward + backward of a stage-1 joint batch (block-diagonal segment mask)",
        "value": round((fwd_ms + bwd_ms) / world, 4), "unit": "ms/batch", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(fwd_ms + bwd_ms, 4), "higher_is_better": False,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded N(0,1))",
        "config": {"workload": "768x1408 joint batch: segments of %s latent frames (images are one frame), "
                               "12 heads, d=128, dense within each segment" % (w.seg_frames,),
                   "name": "joint", "mode": "segment", "l2": "flushed before every timed step (512 MB write)"},
        "per_kernel_ms": {"attn_fwd": round(fwd_ms, 4), "attn_bwd": round(bwd_ms, 4)},
        "roofline": {"bound": "tensor", "kernel": "attn_fwd", "achieved": round(f_tf, 2), "peak": peak,
                     "unit": "TFLOP/s", "frac": round(f_tf / peak, 4), "flops_per_launch": fwd_flops, "traffic": None,
                     "bwd_achieved": round(b_tf, 2), "bwd_frac": round(b_tf / peak, 4)},
        "gpu_launches": 5 * args.steps,
        "clocks": clk,
    }


def _threads():
    try:
        from threadpoolctl import threadpool_info
        n = [p.get("num_threads", 1) for p in threadpool_info()]
        return max(n) if n else os.cpu_count()
    except Exception:
        return os.cpu_count()


def cpu_model() -> str:
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


class CpuMeter:
    """Wall time and the process's CPU time over a region: their ratio is the
    number of cores the oracle actually kept busy (its per-block loops are
    mostly single-threaded numpy; only the products use several BLAS threads)."""

    def __enter__(self):
        self.w0, self.c0 = time.perf_counter(), time.process_time()
        return self

    def __exit__(self, *exc):
        self.wall = time.perf_counter() - self.w0
        self.cpu = time.process_time() - self.c0

    @property
    def cores(self) -> float:
        return round(self.cpu / self.wall, 2) if self.wall > 0 else 1.0


def cpu_baseline(w, x, budget_s=15.0):
    """The fp64 oracle as it stands, on whole heads of the workload until the
    budget is spent; scaled to ms per chunk."""
    from oracle import lcsa_oracle as orc

    done = 0
    streams = [(b, h) for b in range(w.B) for h in range(w.H)]
    with CpuMeter() as meter:
        for b, h in streams:
            orc.lcsa_head(orc.widen(x["q"][b, h]), orc.widen(x["k"][b][h]), orc.widen(x["v"][b][h]),
                          top_k=w.top_k, density=w.density, window=w.window, mode=w.window_mode)
            done += 1
            if time.perf_counter() - meter.w0 > budget_s:
                break
    per_chunk_ms = meter.wall / done * len(streams) / (CHUNKS_PER_STEP.get(w.name, 1) * w.B) * 1e3
    return {"value": round(per_chunk_ms, 2), "unit": UNIT, "cores": meter.cores, "kind": "oracle",
            "threads_available": _threads(), "cpu_model": cpu_model(),
            "sample": "%d of %d (stream, head) units of the workload, whole path (pool, select, "
                      "attention) in fp64, scaled to the full chunk; cores = process CPU time / wall "
                      "time" % (done, len(streams))}


def run_reference(args, world, rank):
    if rank != 0:
        return None
    w = li.workload(args.workload)
    x = li.make_inputs(w)
    from oracle import lcsa_oracle as orc

    units = [(b, h) for b in range(w.B) for h in range(w.H)]
    times = []
    cpu = 0.0
    for i in range(args.warmup + args.steps):
        b, h = units[i % len(units)]
        with CpuMeter() as meter:
            orc.lcsa_head(orc.widen(x["q"][b, h]), orc.widen(x["k"][b][h]), orc.widen(x["v"][b][h]),
                          top_k=w.top_k, density=w.density, window=w.window, mode=w.window_mode)
        if i >= args.warmup:
            times.append(meter.wall)
            cpu += meter.cpu
    per_chunk_ms = statistics.mean(times) * len(units) / (CHUNKS_PER_STEP.get(args.workload, 1) * w.B) * 1e3
    sample = ("one (stream, head) unit per step, whole path (pool, select, attention) in fp64, "
              "scaled by %d units to the full chunk; cores = process CPU time / wall time" % len(units))
    return {
        "impl": "reference", "metric": METRIC, "value": round(per_chunk_ms, 2), "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(statistics.mean(times) * 1e3, 2), "higher_is_better": False,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD_TEXT[args.workload], "name": args.workload},
        "cpu_baseline": {"value": round(per_chunk_ms, 2), "unit": UNIT, "cores": round(cpu / sum(times), 2),
                         "threads_available": _threads(), "cpu_model": cpu_model(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(per_chunk_ms, 2), "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="chunk", choices=sorted(WORKLOAD_TEXT))
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-workloads", action="store_true",
                    help="skip the other configurations (multistream, UHR, clip densities) in the headline line")
    ap.add_argument("--extra-steps", type=int, default=5, help="timed steps per extra configuration")
    ap.add_argument("--mode", default="fwd", choices=["fwd", "bwd", "segment"],
                    help="fwd: the streaming step (default); bwd: the attention backward on a clip; "
                         "segment: stage-1 dense segment attention, forward + backward")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        world = int(os.environ.get("WORLD_SIZE", "1"))
        line = run_reference(args, world, rank)
        if line is not None:
            print(json.dumps(line), flush=True)
        return
    world, rank, local = dist_setup(args.gpus)
    try:
        if args.mode == "bwd":
            if args.workload == "chunk":
                args.workload = "clip"
            line = run_backward(args, world, rank, local)
        elif args.mode == "segment":
            line = run_segment(args, world, rank, local)
        else:
            line = run_ours(args, world, rank, local)
        if rank == 0:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
