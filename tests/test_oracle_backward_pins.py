"""Pins of the oracle's attention gradients (``attend_rows_backward``,
``attend_head_backward``) against things other than their own formulas:
central finite differences of the oracle's forward, torch autograd of a masked
dense attention written independently here, and closed forms that hold for
any input (sum over keys of dk is zero, sum over keys of dv equals the sum of
the output gradients, equal values give zero dq and dk)."""
import math

import numpy as np
import pytest
import torch

import lcsa_inputs as li
from oracle import lcsa_oracle as orc


def _loss_rows(q, k, v, g):
    o, _ = orc.attend_rows(q, k, v)
    return float((o * g).sum())


def test_rows_gradient_matches_central_differences():
    rng = np.random.default_rng(3)
    n, m, d = 5, 9, 8
    q, k, v = rng.standard_normal((n, d)), rng.standard_normal((m, d)), rng.standard_normal((m, d))
    g = rng.standard_normal((n, d))
    dq, dk, dv = orc.attend_rows_backward(q, k, v, g)
    h = 1e-6
    for name, x, grad in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        for _ in range(12):
            i, j = rng.integers(x.shape[0]), rng.integers(d)
            xp, xm = x.copy(), x.copy()
            xp[i, j] += h
            xm[i, j] -= h
            args_p = {"q": q, "k": k, "v": v, name: xp}
            args_m = {"q": q, "k": k, "v": v, name: xm}
            fd = (_loss_rows(args_p["q"], args_p["k"], args_p["v"], g) -
                  _loss_rows(args_m["q"], args_m["k"], args_m["v"], g)) / (2 * h)
            assert abs(fd - grad[i, j]) <= 1e-7 * max(1.0, abs(fd)), (name, i, j, fd, grad[i, j])


def _small_head(frames_q=3, frames_k=5, density=0.5, seed=5):
    w = li.Workload("bwd", B=1, H=1, D=64, Y=16, X=16, q_frames=frames_q, kv_past=(frames_k - frames_q,),
                    cap_frames=frames_k + (frames_k & 1), density=density, seed=seed)
    x = li.make_inputs(w)
    q, k, v = orc.widen(x["q"][0, 0]), orc.widen(x["k"][0][0]), orc.widen(x["v"][0][0])
    ref = orc.lcsa_head(q, k, v, density=density)
    return q, k, v, ref["sel"]


def test_head_gradient_matches_central_differences_with_partial_blocks():
    q, k, v, sel = _small_head()   # 3 query frames, 5 key frames: one-frame oldest blocks
    rng = np.random.default_rng(7)
    g = rng.standard_normal(q.shape)
    dq, dk, dv = orc.attend_head_backward(q, k, v, sel, g)

    def loss(qq, kk, vv):
        o, _ = orc.attend_head(qq, kk, vv, sel)
        return float((o * g).sum())

    h = 1e-6
    for name, x, grad in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        for _ in range(8):
            idx = tuple(rng.integers(s) for s in x.shape)
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            ap = {"q": q, "k": k, "v": v, name: xp}
            am = {"q": q, "k": k, "v": v, name: xm}
            fd = (loss(ap["q"], ap["k"], ap["v"]) - loss(am["q"], am["k"], am["v"])) / (2 * h)
            assert abs(fd - grad[idx]) <= 1e-6 * max(1.0, abs(fd)), (name, idx, fd, grad[idx])


def test_head_gradient_matches_torch_autograd_of_masked_dense_attention():
    q, k, v, sel = _small_head(frames_q=4, frames_k=6, density=0.4, seed=9)
    Tq, Y, X, D = q.shape
    F = k.shape[0]
    # token-level mask written out independently: query token -> its block,
    # key token -> its block, allowed iff the key block is kept for the query block
    def block_of(frames, t, y, x):
        off = frames - 2 * ((frames + 1) // 2)     # -1 when the oldest block has one frame
        return ((t - off) // 2) * (Y // 8) * (X // 8) + (y // 8) * (X // 8) + (x // 8)
    qb = np.array([block_of(Tq, t, y, x) for t in range(Tq) for y in range(Y) for x in range(X)])
    kb = np.array([block_of(F, t, y, x) for t in range(F) for y in range(Y) for x in range(X)])
    mask = np.zeros((qb.size, kb.size), dtype=bool)
    for r in range(qb.size):
        mask[r] = np.isin(kb, sel[qb[r]])
    rng = np.random.default_rng(11)
    g = rng.standard_normal(q.shape)
    tq = torch.tensor(q.reshape(-1, D), requires_grad=True)
    tk = torch.tensor(k.reshape(-1, D), requires_grad=True)
    tv = torch.tensor(v.reshape(-1, D), requires_grad=True)
    s = (tq @ tk.T) / math.sqrt(D)
    s = s.masked_fill(~torch.tensor(mask), float("-inf"))
    o = torch.softmax(s, dim=1) @ tv
    (o * torch.tensor(g.reshape(-1, D))).sum().backward()
    dq, dk, dv = orc.attend_head_backward(q, k, v, sel, g)
    np.testing.assert_allclose(dq.reshape(-1, D), tq.grad.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dk.reshape(-1, D), tk.grad.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dv.reshape(-1, D), tv.grad.numpy(), rtol=1e-10, atol=1e-12)


def test_gradient_closed_forms():
    q, k, v, sel = _small_head(frames_q=2, frames_k=6, density=0.3, seed=13)
    D = q.shape[-1]
    g = np.random.default_rng(17).standard_normal(q.shape)
    dq, dk, dv = orc.attend_head_backward(q, k, v, sel, g)
    # each query row's softmax gradient sums to zero over its keys
    np.testing.assert_allclose(dk.reshape(-1, D).sum(axis=0), 0.0, atol=1e-10)
    # each row's weights sum to one, so the value gradients add up to the output gradients
    np.testing.assert_allclose(dv.reshape(-1, D).sum(axis=0), g.reshape(-1, D).sum(axis=0), rtol=1e-12, atol=1e-10)
    # equal value rows: O does not depend on q or k
    v_eq = np.broadcast_to(v.reshape(-1, D)[0], v.reshape(-1, D).shape).reshape(v.shape).copy()
    dq0, dk0, _ = orc.attend_head_backward(q, k, v_eq, sel, g)
    assert np.abs(dq0).max() < 1e-12 and np.abs(dk0).max() < 1e-12


def test_segment_attention_is_textbook_dense_attention():
    """Within a segment: torch's scaled-dot-product attention (float64, no mask)."""
    rng = np.random.default_rng(21)
    q = rng.standard_normal((3, 8, 8, 16))
    k = rng.standard_normal((3, 8, 8, 16))
    v = rng.standard_normal((3, 8, 8, 16))
    o, lse = orc.segment_attention(q, k, v)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.tensor(q.reshape(1, -1, 16)), torch.tensor(k.reshape(1, -1, 16)), torch.tensor(v.reshape(1, -1, 16)))
    np.testing.assert_allclose(o.reshape(-1, 16), ref[0].numpy(), rtol=1e-12, atol=1e-12)
    s = (q.reshape(-1, 16) @ k.reshape(-1, 16).T) / 4.0
    np.testing.assert_allclose(lse.reshape(-1), np.log(np.exp(s).sum(axis=1)), rtol=1e-12)


def test_segments_equal_block_diagonal_mask_on_a_packed_sequence():
    """Two segments packed into one sequence with a block-diagonal boolean mask
    (torch autograd, float64) give each segment's own attention and gradients."""
    rng = np.random.default_rng(23)
    F = (2, 1)   # a two-frame clip and an image
    segs = [(rng.standard_normal((f, 8, 8, 16)), rng.standard_normal((f, 8, 8, 16)),
             rng.standard_normal((f, 8, 8, 16)), rng.standard_normal((f, 8, 8, 16))) for f in F]
    n = [f * 64 for f in F]
    mask = torch.zeros((sum(n), sum(n)), dtype=torch.bool)
    mask[:n[0], :n[0]] = True
    mask[n[0]:, n[0]:] = True
    tq = torch.tensor(np.concatenate([s[0].reshape(-1, 16) for s in segs]), requires_grad=True)
    tk = torch.tensor(np.concatenate([s[1].reshape(-1, 16) for s in segs]), requires_grad=True)
    tv = torch.tensor(np.concatenate([s[2].reshape(-1, 16) for s in segs]), requires_grad=True)
    g = torch.tensor(np.concatenate([s[3].reshape(-1, 16) for s in segs]))
    sc = (tq @ tk.T / 4.0).masked_fill(~mask, float("-inf"))
    o = torch.softmax(sc, dim=1) @ tv
    (o * g).sum().backward()
    off = 0
    for (q, k, v, do), m in zip(segs, n):
        ro, _ = orc.segment_attention(q, k, v)
        dq, dk, dv = orc.segment_attention_backward(q, k, v, do)
        np.testing.assert_allclose(ro.reshape(-1, 16), o[off:off + m].detach().numpy(), rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(dq.reshape(-1, 16), tq.grad[off:off + m].numpy(), rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(dk.reshape(-1, 16), tk.grad[off:off + m].numpy(), rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(dv.reshape(-1, 16), tv.grad[off:off + m].numpy(), rtol=1e-10, atol=1e-12)
        off += m
