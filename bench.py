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
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained"), "source": "measured"}
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
def run_ours(args, world, rank, local):
    import block_sparse_causal_lcsa_b200 as lc

    w = li.workload(args.workload)
    dev = torch.device("cuda", local)
    peaks = load_peaks()
    # each rank streams an independent video (weak scaling)
    w = rank_workload(w, rank)
    streaming = w.kv_past[0] > 0 or w.B > 1
    x = li.make_inputs(w)
    params = lc.SelectParams(top_k=w.top_k, density=w.density, window=w.window,
                             window_mode=w.window_mode)
    n_chunks = 3
    if streaming:
        cache = lc.KVCache(w.B, w.H, w.cap_frames, w.Y, w.X, w.D, device=dev)
        for b in range(w.B):
            kp = x["k"][b][:, :w.kv_past[b]].unsqueeze(0).to(dev)
            vp = x["v"][b][:, :w.kv_past[b]].unsqueeze(0).to(dev)
            lc.kv_append(cache, kp, vp, lc.pool_qk(kp)[0], stream_offset=b)
        # distinct chunks cycled through the steps (the stream keeps advancing)
        g = torch.Generator().manual_seed(w.seed + 7)
        shp = (w.B, w.H, w.q_frames, w.Y, w.X, w.D)
        chunks = [(x["q"].to(dev),
                   torch.stack([x["k"][b][:, -w.q_frames:] for b in range(w.B)]).to(dev),
                   torch.stack([x["v"][b][:, -w.q_frames:] for b in range(w.B)]).to(dev))]
        for _ in range(n_chunks - 1):
            chunks.append(tuple(torch.randn(shp, generator=g).to(torch.bfloat16).to(dev)
                                for _ in range(3)))
        step = lc.StreamingStep(cache, w.q_frames, params)
        base_state = cache.state()
        tok_window = w.window if w.window_mode >= li.WINDOW_TRUNCATE_TOKENS else 0

        def run_step(i, q=None, k=None, v=None, ev=None):
            if q is None:
                q, k, v = chunks[i % n_chunks]
            # every step sees the workload's cache lengths (host-side state only);
            # the append still writes 2 frames and the pooled K into the ring
            step.cache.set_state(base_state)
            if ev is not None:
                ev[0].record()
            lc.pool_qk(q, None, step.q_pool)
            if ev is not None:
                ev[1].record()
            lc.kv_append(step.cache, k, v)  # pools K while copying it
            if ev is not None:
                ev[2].record()
            lc.select_blocks(step.q_pool, step.q_frames, step.cache, step.params, step.kmax,
                             step.blk_idx, step.blk_cnt, step.workspace)
            if ev is not None:
                ev[3].record()
            lc.sparse_attn_fwd(q, step.cache, step.blk_idx, step.blk_cnt, step.o, step.lse, workspace=step.attn_ws,
                               window=tok_window, window_mode=w.window_mode)
            if ev is not None:
                ev[4].record()
            return step.o

        kernels = ["pool", "kv_append", "select", "attn"]
        q_frames_step = w.q_frames
        sel_ref = step
    else:
        # whole clip: Q, K, V of all frames resident; no append
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
        sel_ws = torch.empty(max(lc.select_workspace_bytes(cache, w.q_frames), 16), dtype=torch.uint8,
                             device=dev)
        attn_ws = lc.attn_workspace(w.D, dev)
        base_state = cache.state()

        class _S:
            pass
        sel_ref = _S()
        sel_ref.blk_idx, sel_ref.blk_cnt, sel_ref.o = blk_idx, blk_cnt, o

        def run_step(i, qq=None, kk=None, vv=None, ev=None):
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

        kernels = ["pool", "select", "attn"]
        q_frames_step = w.q_frames

    # L2 flush: write 512 MB, then read another 256 MB so that the written
    # (dirty) lines are written back before the timed step starts
    flush = torch.empty(512 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
    flush_rd = torch.ones(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)

    def flush_l2():
        flush.zero_()
        flush_rd.sum()

    for i in range(args.warmup):
        flush_l2()
        run_step(i)
    torch.cuda.synchronize()
    if lc.last_device_error() != 0:
        raise RuntimeError("device error during warm-up")

    nev = len(kernels) + 1
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(nev)] for _ in range(args.steps)]
    clocks = ClockSampler(local)
    barrier(world)
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.3)
    t_wall = time.perf_counter()
    for i in range(args.steps):
        flush_l2()
        run_step(args.warmup + i, ev=evs[i])
    torch.cuda.synchronize()
    t_wall = time.perf_counter() - t_wall
    barrier(world)
    time.sleep(0.2)
    clk = clocks.stop()
    if lc.last_device_error() != 0:
        raise RuntimeError("device error during the timed steps")
    step_ms = [evs[i][0].elapsed_time(evs[i][-1]) for i in range(args.steps)]
    per_kernel = {kname: statistics.mean(evs[i][j].elapsed_time(evs[i][j + 1]) for i in range(args.steps))
                  for j, kname in enumerate(kernels)}
    mean_step = statistics.mean(step_ms)
    mean_step_max = max_over_ranks(mean_step, world)
    chunks_per_step = CHUNKS_PER_STEP.get(args.workload, 1) * w.B
    value = whole_job_ms_per_chunk(mean_step_max, chunks_per_step, world)

    flops = attn_flops(sel_ref.blk_cnt, sel_ref.blk_idx, cache, w.Hb, w.Wb, w.D)
    attn_s = per_kernel["attn"] / 1e3
    achieved_tflops = flops / attn_s / 1e12
    peak = peaks["bf16_tflops"]

    # e2e: the same step through the API with inputs from pinned host memory and
    # the output read back, copies inside the timed region
    e2e = None
    if streaming:
        # chunks from pinned host memory through lc.HostPipeline: each chunk's
        # inputs cross PCIe while the previous chunk computes, and its O comes
        # back on a third stream; the timed region runs from the first timed
        # chunk's host-to-device copy to the last chunk's device-to-host copy
        hq = chunks[0][0].cpu().pin_memory()
        hk = chunks[0][1].cpu().pin_memory()
        hv = chunks[0][2].cpu().pin_memory()
        ho = torch.empty(hq.shape, dtype=torch.bfloat16).pin_memory()
        pipe = lc.HostPipeline(step)
        e_start = torch.cuda.Event(enable_timing=True)
        done = None
        for i in range(args.warmup + args.steps):
            if i == args.warmup:
                torch.cuda.synchronize()
                e_start.record(pipe.h2d_stream)
            flush_l2()
            step.cache.set_state(base_state)
            done = pipe.submit(hq, hk, hv, ho)
        torch.cuda.synchronize()
        e2e_ms = e_start.elapsed_time(done) / args.steps
        e2e_ms = max_over_ranks(e2e_ms, world)
        e2e = {"value": whole_job_ms_per_chunk(e2e_ms, chunks_per_step, world), "unit": UNIT,
               "h2d_bytes_per_step": hq.numel() * 2 + hk.numel() * 2 + hv.numel() * 2,
               "d2h_bytes_per_step": ho.numel() * 2,
               "pipelined": "copies of chunk i+1 overlap the compute of chunk i (lc.HostPipeline)"}
    else:
        hq = q.cpu().pin_memory()
        hk = k.cpu().pin_memory()
        hv = v.cpu().pin_memory()
        ho = torch.empty(hq.shape, dtype=torch.bfloat16).pin_memory()
        e_start = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
        e_end = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
        for i in range(args.warmup + args.steps):
            if i >= args.warmup:
                e_start[i - args.warmup].record()
            q.copy_(hq, non_blocking=True)
            k.copy_(hk, non_blocking=True)
            v.copy_(hv, non_blocking=True)
            out = run_step(i)
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

    # the same step replayed from a CUDA graph (one launch per step), inputs in
    # the graph's static buffers, L2 flushed outside the timed events
    graph = None
    if streaming:
        step.cache.set_state(base_state)
        step.graph_step(*chunks[0])
        g_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
        for i in range(args.warmup + args.steps):
            flush_l2()
            step.cache.set_state(base_state)
            if i >= args.warmup:
                g_ev[i - args.warmup][0].record()
            step.graph_step()
            if i >= args.warmup:
                g_ev[i - args.warmup][1].record()
        torch.cuda.synchronize()
        if lc.last_device_error() != 0:
            raise RuntimeError("device error during the graph steps")
        g_ms = max_over_ranks(statistics.mean(a.elapsed_time(b) for a, b in g_ev), world)
        graph = {"ms_per_chunk": round(whole_job_ms_per_chunk(g_ms, chunks_per_step, world), 4),
                 "graph_launches_per_step": 1}

    # HBM-side kernels: algorithmic bytes per launch
    tokens_q = w.B * w.H * q_frames_step * w.Y * w.X
    if "kv_append" in per_kernel:
        # pool reads Q (bf16) once and writes one float64 row per block; the
        # append reads the new K and V once, writes them into the ring and
        # writes K's pooled rows
        bytes_pool = tokens_q * w.D * 2 + (tokens_q // 128) * w.D * 8
        bytes_app = 2 * (2 * tokens_q * w.D * 2) + (tokens_q // 128) * w.D * 8
        hbm = {"pool_gbs": bytes_pool / (per_kernel["pool"] / 1e3) / 1e9,
               "kv_append_gbs": bytes_app / (per_kernel["kv_append"] / 1e3) / 1e9}
    else:
        # whole clip: pool reads Q and K once and writes their pooled rows
        bytes_pool = 2 * tokens_q * w.D * 2 + 2 * (tokens_q // 128) * w.D * 8
        hbm = {"pool_gbs": bytes_pool / (per_kernel["pool"] / 1e3) / 1e9}

    traffic = None
    tfile = os.path.join(ROOT, "profiles", "attn_fwd_%s.traffic.txt" % args.workload)
    if os.path.exists(tfile):
        rec = dict(line.split(":", 1) for line in open(tfile) if ":" in line and not line.startswith("#"))
        if rec.get("source_hash", "").strip() == attn_source_hash():
            traffic = int(rec["bytes_per_launch"])

    # kernels per timed step: the ingest (streaming graph: Q pooling and the
    # fused K/V append in one launch; clip: Q and K pooling), score + top-K, the
    # attention and, when its last wave is split, the merge of the halves
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    units = w.B * w.H * ((w.q_frames + 1) // 2) * w.Hb * w.Wb
    split = units > sms and 0 < units % sms <= sms // 2
    launches_per_step = 1 + 2 + (2 if split else 1)
    # the headline is the step as a user runs it in production: replayed from a
    # CUDA graph (same kernels, same work, one launch); the eager run with CUDA
    # events between the kernels gives the per-kernel split
    eager_value = value
    step_ms = mean_step_max
    if graph is not None:
        value = graph["ms_per_chunk"]
        step_ms = value * chunks_per_step * world
    line = {
        "metric": METRIC, "value": round(value, 4), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(step_ms, 4),
        "eager_ms_per_chunk": round(eager_value, 4),
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
        "sparse_attn_tflops": round(achieved_tflops, 2),
        "roofline": {"bound": "tensor", "kernel": "attn_fwd", "achieved": round(achieved_tflops, 2),
                     "peak": peak, "unit": "TFLOP/s", "frac": round(achieved_tflops / peak, 4),
                     "peak_source": "%s bf16 burst (MEASURED_PEAKS.json)" % peaks["source"],
                     "flops_per_launch": flops, "traffic": traffic},
        "hbm_kernels": {k2: round(v2, 1) for k2, v2 in hbm.items()},
        "cuda_graph": graph,
        "hbm_peak_gbs": peaks["hbm_gbs"],
        "e2e": e2e,
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clk,
        "wall_s_timed": round(t_wall, 4),
    }
    if rank == 0 and not args.no_cpu_baseline and world == 1:
        line["cpu_baseline"] = cpu_baseline(w, x, budget_s=args.cpu_budget)
    return line


# ----------------------------------------------------------------------------- oracle arm
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
    d_o = torch.randn(q.shape, generator=g).to(torch.bfloat16).to(dev)
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
        from oracle import lcsa_oracle as orc
        t0 = time.perf_counter()
        h = 0
        qh, kh, vh = orc.widen(x["q"][0, h]), orc.widen(x["k"][0][h]), orc.widen(x["v"][0][h])
        sel = [idx[0, h, i, :int(cnt[0, h, i])].cpu().numpy() for i in range(cnt.shape[2])]
        # a bounded sample: the first query blocks of one head, scaled by their share of the kept pairs
        n_rows = 0
        kept = 0
        Tq, Y, X, D = qh.shape
        for i in range(len(sel)):
            qidx = orc.block_token_index(Tq, Y, X, [i])
            kidx = orc.block_token_index(kh.shape[0], Y, X, sel[i])
            orc.attend_rows_backward(qh.reshape(-1, D)[qidx], kh.reshape(-1, D)[kidx], vh.reshape(-1, D)[kidx],
                                     orc.widen(d_o[0, h].cpu()).reshape(-1, D)[qidx])
            n_rows += 1
            kept += len(sel[i])
            if time.perf_counter() - t0 > args.cpu_budget:
                break
        el = time.perf_counter() - t0
        total_kept = int(cnt.sum().item())
        cpu_ms = el / kept * total_kept * 1e3
        line["cpu_baseline"] = {"value": round(cpu_ms, 1), "unit": "ms/clip", "cores": _threads(), "kind": "oracle",
                                "sample": "%d query blocks (%d kept block pairs) of head 0, attend_rows_backward "
                                          "in fp64, scaled by kept pairs to all %d" % (n_rows, kept, total_kept)}
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


def cpu_baseline(w, x, budget_s=15.0):
    """The fp64 oracle as it stands, on whole heads of the workload until the
    budget is spent; scaled to ms per chunk."""
    from oracle import lcsa_oracle as orc

    t0 = time.perf_counter()
    done = 0
    streams = [(b, h) for b in range(w.B) for h in range(w.H)]
    for b, h in streams:
        orc.lcsa_head(orc.widen(x["q"][b, h]), orc.widen(x["k"][b][h]), orc.widen(x["v"][b][h]),
                      top_k=w.top_k, density=w.density, window=w.window, mode=w.window_mode)
        done += 1
        if time.perf_counter() - t0 > budget_s:
            break
    el = time.perf_counter() - t0
    per_chunk_ms = el / done * len(streams) / (CHUNKS_PER_STEP.get(w.name, 1) * w.B) * 1e3
    return {"value": round(per_chunk_ms, 2), "unit": UNIT, "cores": _threads(), "kind": "oracle",
            "sample": "%d of %d (stream, head) units of the workload, whole path (pool, select, "
                      "attention) in fp64, scaled to the full chunk" % (done, len(streams))}


def run_reference(args, world, rank):
    if rank != 0:
        return None
    w = li.workload(args.workload)
    x = li.make_inputs(w)
    from oracle import lcsa_oracle as orc

    units = [(b, h) for b in range(w.B) for h in range(w.H)]
    times = []
    for i in range(args.warmup + args.steps):
        b, h = units[i % len(units)]
        t0 = time.perf_counter()
        orc.lcsa_head(orc.widen(x["q"][b, h]), orc.widen(x["k"][b][h]), orc.widen(x["v"][b][h]),
                      top_k=w.top_k, density=w.density, window=w.window, mode=w.window_mode)
        if i >= args.warmup:
            times.append(time.perf_counter() - t0)
    per_chunk_ms = statistics.mean(times) * len(units) / (CHUNKS_PER_STEP.get(args.workload, 1) * w.B) * 1e3
    sample = ("one (stream, head) unit per step, whole path (pool, select, attention) in fp64, "
              "scaled by %d units to the full chunk" % len(units))
    return {
        "impl": "reference", "metric": METRIC, "value": round(per_chunk_ms, 2), "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(statistics.mean(times) * 1e3, 2), "higher_is_better": False,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD_TEXT[args.workload], "name": args.workload},
        "cpu_baseline": {"value": round(per_chunk_ms, 2), "unit": UNIT, "cores": _threads(),
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
