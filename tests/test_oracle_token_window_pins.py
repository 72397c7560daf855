"""Pins of the oracle's token-level locality window (``token_window_range``,
``token_block_range``, the masked attention in ``attend_head``) against hand
values, brute force over every (query token, key token) pair with a torch
masked softmax written here, and invariants (a window covering the frame is no
window; empty rows give O = 0, LSE = -inf)."""
import math

import numpy as np
import torch

import lcsa_inputs as li
from oracle import lcsa_oracle as orc

T, P = orc.WINDOW_TRUNCATE_TOKENS, orc.WINDOW_PRESERVE_TOKENS


def test_hand_values():
    # 96 tokens, a 72-token window: the query sits at offset 36
    assert orc.token_window_range(0, 96, 72, T) == (0, 36)
    assert orc.token_window_range(50, 96, 72, T) == (14, 86)
    assert orc.token_window_range(95, 96, 72, T) == (59, 96)
    assert orc.token_window_range(0, 96, 72, P) == (0, 72)
    assert orc.token_window_range(90, 96, 72, P) == (24, 96)
    assert orc.token_window_range(40, 48, 72, P) == (0, 48)     # window wider than the frame
    # block 6 (tokens 48..55): windows from [12, 84) to [19, 91) -> blocks 1..11
    assert orc.token_block_range(6, 96, 72, T) == (1, 12)
    assert orc.token_block_range(0, 96, 72, P) == (0, 9)
    assert orc.token_block_range(11, 96, 72, P) == (3, 12)


def _head(Y=24, X=32, frames=4, window=20, mode=T, density=0.6, seed=3):
    w = li.Workload("tw", B=1, H=1, D=64, Y=Y, X=X, q_frames=2, kv_past=(frames - 2,), cap_frames=frames,
                    density=density, seed=seed)
    x = li.make_inputs(w)
    return orc.widen(x["q"][0, 0]), orc.widen(x["k"][0][0]), orc.widen(x["v"][0][0])


def test_brute_force_token_mask_with_torch():
    for mode in (T, P):
        q, k, v = _head(mode=mode)
        Tq, Y, X, D = q.shape
        F = k.shape[0]
        W = 20
        ref = orc.lcsa_head(q, k, v, density=0.6, window=W, mode=mode)
        # every key token's block id and coordinates, written out independently
        Hb, Wb = Y // 8, X // 8
        def bid(frames, t, y, x):
            off = frames - 2 * ((frames + 1) // 2)
            return ((t - off) // 2) * Hb * Wb + (y // 8) * Wb + (x // 8)
        kt = [(t, y, x) for t in range(F) for y in range(Y) for x in range(X)]
        qt = [(t, y, x) for t in range(Tq) for y in range(Y) for x in range(X)]
        half = W // 2
        def win(c, n):
            s = c - half
            if mode == T:
                return max(0, s), min(n, s + W)
            st = max(0, min(s, n - W))
            return st, min(n, st + W)
        mask = np.zeros((len(qt), len(kt)), dtype=bool)
        for a, (t, y, x) in enumerate(qt):
            kept = set(ref["sel"][bid(Tq, t, y, x)].tolist())
            y0, y1 = win(y, Y)
            x0, x1 = win(x, X)
            for c, (tk, yk, xk) in enumerate(kt):
                mask[a, c] = bid(F, tk, yk, xk) in kept and y0 <= yk < y1 and x0 <= xk < x1
        s = torch.tensor(q.reshape(-1, D)) @ torch.tensor(k.reshape(-1, D)).T / math.sqrt(D)
        s = s.masked_fill(~torch.tensor(mask), float("-inf"))
        o = torch.softmax(s, dim=1) @ torch.tensor(v.reshape(-1, D))
        np.testing.assert_allclose(ref["O"].reshape(-1, D), o.numpy(), rtol=1e-10, atol=1e-12)
        # candidates: a block is allowed iff some token of the query block sees some token of it
        C_bf = []
        for i in range(Hb * Wb):
            yb, xb = divmod(i, Wb)
            ys = set()
            xs = set()
            for yy in range(8 * yb, 8 * yb + 8):
                a, b = win(yy, Y)
                ys |= {c // 8 for c in range(a, b)}
            for xx in range(8 * xb, 8 * xb + 8):
                a, b = win(xx, X)
                xs |= {c // 8 for c in range(a, b)}
            C_bf.append(len(ys) * len(xs) * ((F + 1) // 2))
        assert list(ref["C"][-Hb * Wb:]) == C_bf


def test_window_covering_the_frame_is_no_window():
    q, k, v = _head(Y=16, X=24)
    a = orc.lcsa_head(q, k, v, density=0.5, window=64, mode=T)
    b = orc.lcsa_head(q, k, v, density=0.5)
    for s1, s2 in zip(a["sel"], b["sel"]):
        assert np.array_equal(s1, s2)
    np.testing.assert_allclose(a["O"], b["O"], rtol=1e-12, atol=1e-14)


def test_empty_rows_give_zero_output():
    # a 2-token window and one kept block: most query tokens see none of it
    q, k, v = _head(Y=16, X=16, frames=2, density=0.0)
    ref = orc.lcsa_head(q, k, v, top_k=1, window=2, mode=T)
    L = ref["LSE"].reshape(-1)
    O = ref["O"].reshape(-1, q.shape[-1])
    empty = ~np.isfinite(L)
    assert empty.any() and (~empty).any()
    assert np.all(O[empty] == 0.0)
    assert np.all(np.isfinite(O))
