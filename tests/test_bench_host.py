"""Host-side arithmetic behind bench.py's JSON line (no GPU): the FLOP count
that the roofline divides by, and the whole-job throughput across ranks."""
import importlib.util
import os

import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


class _Cache:
    """Just the cache state attn_flops reads: the first cached frame of each stream."""

    def __init__(self, begins):
        self._begins = begins

    def begin(self, b):
        return self._begins[b]


def test_attn_flops_counts_kept_key_tokens():
    bench = _bench()
    Hb, Wb, D = 2, 3, 128
    # one stream, one head, two query blocks keeping 3 and 2 blocks (-1 = unused slot)
    cnt = torch.tensor([[[3, 2]]], dtype=torch.int32)
    idx = torch.tensor([[[[0, 4, 7], [2, 9, -1]]]], dtype=torch.int32)
    full = bench.attn_flops(cnt, idx, _Cache([4]), Hb, Wb, D)
    assert full == 4.0 * D * 128 * (5 * 128)
    # an odd first cached frame leaves the oldest key block (ids < Hb*Wb) with one
    # frame: kept blocks 0, 4 and 2 then hold 64 keys each; the -1 slot is not counted
    partial = bench.attn_flops(cnt, idx, _Cache([3]), Hb, Wb, D)
    assert partial == 4.0 * D * 128 * (5 * 128 - 3 * 64)


def test_attn_flops_sums_streams_separately():
    bench = _bench()
    cnt = torch.tensor([[[1]], [[1]]], dtype=torch.int32)
    idx = torch.tensor([[[[0]]], [[[0]]]], dtype=torch.int32)
    # stream 0 starts on an even frame (full block), stream 1 on an odd one (one frame)
    f = bench.attn_flops(cnt, idx, _Cache([2, 1]), 1, 1, 64)
    assert f == 4.0 * 64 * 128 * (128 + 64)


def test_whole_job_throughput_divides_by_every_rank_chunk():
    bench = _bench()
    # 4 ranks, 13 chunks each, slowest rank 26 ms: 0.5 ms per chunk of the whole job
    assert bench.whole_job_ms_per_chunk(26.0, 13, 4) == 0.5
    assert bench.whole_job_ms_per_chunk(0.25, 1, 1) == 0.25


class _CacheSpan:
    """begin / end frames per stream, as bench.allowed_pairs reads them."""

    def __init__(self, spans):
        self._s = spans

    def begin(self, b):
        return self._s[b][0]

    def end(self, b):
        return self._s[b][1]


def test_allowed_pairs_equals_the_oracles_candidate_counts():
    """The selection's float64 work is counted from the pairs the coarse map
    scores; for every window mode that count equals the sum of the oracle's
    per-row candidate counts C_i."""
    import numpy as np
    import lcsa_inputs as li
    from oracle import lcsa_oracle as orc

    bench = _bench()
    w = li.workload("chunk")
    assert bench.allowed_pairs(w, _CacheSpan([(0, 6)])) == 12 * 66 * 198
    for window, mode in [(0, 0), (3, 0), (3, 1), (5, 0), (20, 2), (20, 3), (35, 2)]:
        w = li.Workload("pairs", B=2, H=1, D=64, Y=40, X=56, q_frames=2, kv_past=(4, 3), cap_frames=6,
                        density=0.2, window=window, window_mode=mode, seed=3)
        spans = [(0, 6), (1, 6)]
        got = bench.allowed_pairs(w, _CacheSpan(spans))
        want = 0
        for lo, hi in spans:
            F = hi - lo
            nKT = (F + 1) // 2
            qp = np.zeros((w.Hb * w.Wb, w.D))
            kp = np.zeros((nKT * w.Hb * w.Wb, w.D))
            _, _, Cs = orc.select_head(qp, kp, w.q_frames, F, w.Y, w.X, density=w.density,
                                       window=window, mode=mode)
            want += int(Cs.sum())
        assert got == want, (window, mode, got, want)


def test_reference_arm_prints_the_contract_line():
    """bench.py --impl reference times the oracle on host cores and prints the
    same JSON line as the GPU arm: the same metric, unit and workload text,
    time-like (lower is better), an e2e that moves no bytes between host and
    device, and a cpu_baseline describing this run. Under several ranks, rank 0
    alone runs it; the others return without work."""
    import argparse
    import json

    b = _bench()
    args = argparse.Namespace(workload="chunk", steps=1, warmup=0)
    assert b.run_reference(args, 2, 1) is None
    line = b.run_reference(args, 1, 0)
    json.dumps(line)
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["metric"] == b.METRIC and line["unit"] == b.UNIT
    assert line["config"]["workload"] == b.WORKLOAD_TEXT["chunk"]
    assert line["higher_is_better"] is False and line["value"] > 0 and line["steps"] == 1
    assert line["e2e"] == {"value": line["value"], "unit": b.UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == line["value"] and cb["cores"] > 0 and cb["sample"]


def test_backward_cpu_baseline_selects_with_the_oracle():
    """The backward mode's CPU baseline runs on host inputs alone: the oracle
    selects its own blocks, and the kept-pair total it scales by equals every
    head's own count times the heads (K_i depends only on the geometry)."""
    import lcsa_inputs as li
    from oracle import lcsa_oracle as orc

    b = _bench()
    w = li.small_variant(li.workload("clip"), H=2, Y=16, X=24)
    x = li.make_inputs(w)
    d_o = torch.randn(x["q"].shape, generator=torch.Generator().manual_seed(3)).to(torch.bfloat16)
    cb = b.backward_cpu_baseline(w, x, d_o, budget_s=1.0)
    assert cb["kind"] == "oracle" and cb["value"] > 0 and cb["unit"] == "ms/clip" and cb["cores"] > 0
    assert w.B == 1
    for h in range(w.H):
        qh, kh = orc.widen(x["q"][0, h]), orc.widen(x["k"][0][h])
        _, Ks, _ = orc.select_head(orc.pool_blocks(qh), orc.pool_blocks(kh), qh.shape[0], kh.shape[0], w.Y, w.X,
                                   w.top_k, w.density, w.window, w.window_mode)
        assert int(Ks.sum()) * w.H == cb["kept_pairs_total"]
