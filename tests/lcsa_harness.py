"""Shared helpers of the GPU parity tests: run a workload through the C ABI and
the same workload through the fp64 oracle, then compare."""
from __future__ import annotations

import numpy as np
import torch

import lcsa_inputs as li
from oracle import lcsa_oracle as orc

ATOL = 2e-2     # max-abs error of O against fp64 (bf16 inputs, fp32 accumulation)
RTOL_L2 = 1e-2  # relative L2 error of O against fp64
LSE_ATOL = 2e-3


def build_cache(lc, w: li.Workload, x, dev, chunked_past: bool = True):
    """Fill a cache the streaming way: each stream's past frames, then the
    current chunk of all streams in one append. Returns (cache, k_new, v_new)."""
    cache = lc.KVCache(w.B, w.H, w.cap_frames, w.Y, w.X, w.D, device=dev)
    for b in range(w.B):
        past = w.kv_past[b]
        if past == 0:
            continue
        kp = x["k"][b][:, :past].unsqueeze(0).to(dev)
        vp = x["v"][b][:, :past].unsqueeze(0).to(dev)
        if chunked_past and past % 2 == 0 and past > 2:
            for f in range(0, past, 2):  # two frames at a time, like a live stream
                kc, vc = kp[:, :, f:f + 2].contiguous(), vp[:, :, f:f + 2].contiguous()
                lc.kv_append(cache, kc, vc, lc.pool_qk(kc)[0], stream_offset=b)
        else:
            lc.kv_append(cache, kp, vp, lc.pool_qk(kp)[0], stream_offset=b)
    k_new = torch.stack([x["k"][b][:, -w.q_frames:] for b in range(w.B)]).to(dev)
    v_new = torch.stack([x["v"][b][:, -w.q_frames:] for b in range(w.B)]).to(dev)
    return cache, k_new, v_new


def params_of(lc, w: li.Workload):
    return lc.SelectParams(top_k=w.top_k, density=w.density, window=w.window,
                           window_mode=w.window_mode)


def run_gpu(lc, w: li.Workload, x, dev="cuda"):
    """One streaming step of workload w on the GPU; returns host copies."""
    cache, k_new, v_new = build_cache(lc, w, x, dev)
    step = lc.StreamingStep(cache, w.q_frames, params_of(lc, w))
    q = x["q"].to(dev)
    o, lse = step(q, k_new, v_new)
    torch.cuda.synchronize()
    err = lc.last_device_error()
    return {
        "cache": cache, "step": step, "q": q, "err": err,
        "q_pool": step.q_pool.cpu().numpy(), "k_pool_ring": cache.k_pool.cpu().numpy(),
        "blk_idx": step.blk_idx.cpu().numpy(), "blk_cnt": step.blk_cnt.cpu().numpy(),
        "O": o.double().cpu().numpy(), "LSE": lse.double().cpu().numpy(),
    }


def ring_to_logical(cache, k_pool_ring: np.ndarray, b: int, h: int) -> np.ndarray:
    """Pooled K of stream b, head h in logical block order (oldest first)."""
    m0 = cache.begin(b) // 2
    nKT = cache.end(b) // 2 - m0
    cap_blk = cache.cap_frames // 2
    rows = [k_pool_ring[b, h, (m0 + t) % cap_blk] for t in range(nKT)]
    return np.stack(rows).reshape(-1, cache.D)


def oracle_head(w: li.Workload, x, b: int, h: int, rows=None):
    return orc.lcsa_head(orc.widen(x["q"][b, h]), orc.widen(x["k"][b][h]), orc.widen(x["v"][b][h]),
                         top_k=w.top_k, density=w.density, window=w.window, mode=w.window_mode,
                         rows=rows)


def check_selection(got_idx, got_cnt, sel, where=""):
    assert got_cnt.shape[0] == len(sel)
    for i, s in enumerate(sel):
        c = int(got_cnt[i])
        assert c == len(s), "%s row %d: K %d vs %d" % (where, i, c, len(s))
        assert np.array_equal(got_idx[i, :c], s), "%s row %d: %s vs %s" % (
            where, i, got_idx[i, :c].tolist(), s.tolist())
        assert (got_idx[i, c:] == -1).all()


def o_errors(got: np.ndarray, ref: np.ndarray):
    mask = ~np.isnan(ref)
    d = got[mask] - ref[mask]
    return float(np.abs(d).max()), float(np.linalg.norm(d) / np.linalg.norm(ref[mask]))


def check_output(got_o, ref_o, got_lse=None, ref_lse=None, where=""):
    mx, rel = o_errors(got_o, ref_o)
    assert mx <= ATOL and rel <= RTOL_L2, "%s O max-abs %.3g rel-L2 %.3g" % (where, mx, rel)
    if got_lse is not None:
        m = ~np.isnan(ref_lse)
        le = float(np.abs(got_lse[m] - ref_lse[m]).max())
        assert le <= LSE_ATOL, "%s LSE max-abs %.3g" % (where, le)
    return mx, rel


def compare_all(w: li.Workload, x, g, heads=None, o_rows=None):
    """Bitwise pooled features and selections of the given heads (default
    all); O and LSE on the given query blocks (default all)."""
    for b in range(w.B):
        for h in (range(w.H) if heads is None else heads):
            ref = oracle_head(w, x, b, h, rows=o_rows)
            where = "%s b%d h%d" % (w.name, b, h)
            assert np.array_equal(g["q_pool"][b, h].reshape(-1, w.D), ref["q_pool"]), where + " q_pool"
            assert np.array_equal(ring_to_logical(g["cache"], g["k_pool_ring"], b, h),
                                  ref["k_pool"]), where + " k_pool"
            check_selection(g["blk_idx"][b, h], g["blk_cnt"][b, h], ref["sel"], where)
            check_output(g["O"][b, h], ref["O"], g["LSE"][b, h], ref["LSE"], where)
