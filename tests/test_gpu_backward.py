"""GPU parity of the attention gradients (lcsa_sparse_attn_bwd) against the
fp64 oracle's attend_head_backward. The oracle works from the host inputs
alone: it pools and selects its own blocks, and each case first checks that
the library attended exactly those blocks over the same cached key frames.

Tolerance (derived from the arithmetic): Q, K, V, dO are bf16 and exact in
both paths; the GPU rounds P and dS to bf16 (relative error 2^-9) before their
tensor-core products, accumulates in fp32 and rounds dQ, dK, dV to bf16
(2^-9). Summed over hundreds to thousands of keys these independent rounding
errors give a relative L2 error of a few 1e-3 (measured on these cases: at
most 3.3e-3 rel-L2 and 5.5e-3 max-abs over the tensor's largest magnitude);
the bar is rel-L2 <= 5e-3 per tensor, with max-abs <= 1e-2 of the tensor's
largest magnitude, so a change that doubled the gradient error fails."""
import numpy as np
import pytest
import torch

import lcsa_inputs as li
from lcsa_harness import check_selection, oracle_head
from oracle import lcsa_oracle as orc

pytestmark = pytest.mark.gpu

REL_L2 = 5e-3
MAX_REL = 1e-2


@pytest.fixture(scope="module")
def lc():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import block_sparse_causal_lcsa_b200 as m
    return m


def _errs(got, ref):
    d = got - ref
    scale = max(np.abs(ref).max(), 1e-30)
    return float(np.linalg.norm(d) / max(np.linalg.norm(ref), 1e-30)), float(np.abs(d).max() / scale)


def _check(got, ref, where):
    rel, mx = _errs(got, ref)
    print("%s rel-L2 %.3g max-abs/max %.3g" % (where, rel, mx))
    assert rel <= REL_L2 and mx <= MAX_REL, "%s rel-L2 %.3g max-abs/max %.3g" % (where, rel, mx)
    return rel, mx


def _run(lc, w, x, seed=1):
    """Forward + backward on the GPU. The queries are the newest q_frames
    frames of each stream's cache; with no past frames (the clip workloads)
    the key timeline is the query timeline, the training form."""
    from lcsa_harness import build_cache
    dev = "cuda"
    cache, k_new, v_new = build_cache(lc, w, x, dev)
    lc.kv_append(cache, k_new, v_new)
    q = x["q"].to(dev)
    params = lc.SelectParams(top_k=w.top_k, density=w.density, window=w.window, window_mode=w.window_mode)
    q_pool = lc.pool_qk(q)[0]
    idx, cnt = lc.select_blocks(q_pool, w.q_frames, cache, params)
    o, lse = lc.sparse_attn_fwd(q, cache, idx, cnt)
    g = torch.Generator().manual_seed(seed)
    d_o_host = torch.randn(q.shape, generator=g).to(torch.bfloat16)
    dq, dk, dv = lc.sparse_attn_bwd(q, cache, idx, cnt, o, lse, d_o_host.to(dev))
    torch.cuda.synchronize()
    assert lc.last_device_error() == 0
    return cache, q, idx, cnt, d_o_host, dq, dk, dv


def _oracle_grads(w, x, d_o, b, h):
    """Stream b, head h through the oracle from the host inputs alone: its own
    selection, the key timeline, and dq, dk, dv over that timeline."""
    ref = oracle_head(w, x, b, h, rows=[])    # pooling and selection; no forward rows
    kh, vh = orc.widen(x["k"][b][h]), orc.widen(x["v"][b][h])
    rq, rk, rv = orc.attend_head_backward(orc.widen(x["q"][b, h]), kh, vh, ref["sel"], orc.widen(d_o[b, h]))
    return ref["sel"], kh, rq, rk, rv


def _logical(cache, t, b, h):
    """Frames [begin, end) of stream b, head h of a ring tensor, oldest first."""
    lo, hi = cache.state()[b]
    return torch.stack([t[b, h, f % cache.cap_frames] for f in range(lo, hi)]).double().cpu().numpy()


def _compare(lc, w, x, heads=None):
    cache, q, idx, cnt, d_o, dq, dk, dv = _run(lc, w, x)
    worst = [0.0, 0.0, 0.0]
    for b in range(w.B):
        for h in (range(w.H) if heads is None else heads):
            where = "%s b%d h%d" % (w.name, b, h)
            sel, kh, rq, rk, rv = _oracle_grads(w, x, d_o, b, h)
            # the library attended the oracle's blocks over the same key frames
            check_selection(idx[b, h].cpu().numpy(), cnt[b, h].cpu().numpy(), sel, where)
            assert np.array_equal(_logical(cache, cache.k, b, h), kh), where + " cached K"
            e = [_check(dq[b, h].double().cpu().numpy(), rq, where + " dq")[0],
                 _check(_logical(cache, dk, b, h), rk, where + " dk")[0],
                 _check(_logical(cache, dv, b, h), rv, where + " dv")[0]]
            worst = [max(a, c) for a, c in zip(worst, e)]
    return worst


TRAIN = [
    li.workload("tiny"),
    li.small_variant(li.workload("clip"), H=2, Y=16, X=24),                    # 26 frames, block-causal
    li.small_variant(li.workload("clip"), H=1, Y=16, X=16, q_frames=7, cap_frames=8),  # odd: one-frame oldest block
    li.small_variant(li.workload("clip_30"), H=1, Y=24, X=16, D=64, q_frames=10, cap_frames=10),
]


@pytest.mark.parametrize("w", TRAIN, ids=[w.name + "_%df" % w.q_frames for w in TRAIN])
def test_training_gradients_every_element(lc, w):
    x = li.make_inputs(w)
    print("worst rel-L2 dq/dk/dv", _compare(lc, w, x))


STREAM = [
    li.small_variant(li.workload("chunk"), H=2, Y=24, X=40),
    li.small_variant(li.workload("multistream"), H=2, Y=16, X=24),
    li.Workload("odd_stream", B=1, H=2, D=128, Y=16, X=16, q_frames=2, kv_past=(1,), cap_frames=4, density=0.5, seed=33),
]


@pytest.mark.parametrize("w", STREAM, ids=[w.name for w in STREAM])
def test_streaming_gradients_every_element(lc, w):
    """Queries = the newest frames of each stream's cache (ragged streams, a
    one-frame query block, a one-frame oldest key block)."""
    x = li.make_inputs(w)
    _compare(lc, w, x)


def test_full_size_chunk_gradients_two_heads(lc):
    w = li.workload("chunk")
    x = li.make_inputs(w)
    _compare(lc, w, x, heads=[0, w.H - 1])


def test_backward_is_deterministic(lc):
    w = li.small_variant(li.workload("clip"), H=2, Y=16, X=24)
    x = li.make_inputs(w)
    a = _run(lc, w, x)
    b = _run(lc, w, x)
    for u, v in zip(a[5:], b[5:]):
        assert torch.equal(u, v)
