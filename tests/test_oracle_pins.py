"""Pins of the fp64 oracle against things other than itself.

Each test checks the oracle against exact rational arithmetic, a brute-force
enumeration, a hand-derived fixture, a closed form, or a library routine
(torch's scaled-dot-product attention in float64), chosen so that a dropped
term, a wrong index or a transposed operand anywhere in the oracle fails one
of them. No test here needs a GPU.
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle import lcsa_oracle as orc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _bf16_array(shape, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(shape, generator=g) * scale).to(torch.bfloat16).double().numpy()


def _tblk(f, F):
    # temporal block of frame f when 2-frame blocks are counted back from frame F-1
    return (f + F % 2) // 2


# ----------------------------------------------------------------------------- geometry
def test_temporal_blocks_hand_cases():
    assert orc.temporal_blocks(1) == [[0]]
    assert orc.temporal_blocks(2) == [[0, 1]]
    assert orc.temporal_blocks(3) == [[0], [1, 2]]
    assert orc.temporal_blocks(6) == [[0, 1], [2, 3], [4, 5]]
    assert orc.temporal_blocks(7) == [[0], [1, 2], [3, 4], [5, 6]]
    for F in range(1, 12):
        for t, frames in enumerate(orc.temporal_blocks(F)):
            assert all(_tblk(f, F) == t for f in frames)


# ----------------------------------------------------------------------------- pooling
@pytest.mark.parametrize("F", [2, 3])
def test_pool_equals_exact_rational_mean(F):
    Y, X, D = 16, 8, 3
    x = _bf16_array((F, Y, X, D), seed=10 + F)
    got = orc.pool_blocks(x)
    nT, Hb, Wb = (F + 1) // 2, Y // 8, X // 8
    sums = {}
    for f in range(F):
        for y in range(Y):
            for xx in range(X):
                j = _tblk(f, F) * Hb * Wb + (y // 8) * Wb + (xx // 8)
                acc = sums.setdefault(j, [[Fraction(0)] * D, 0])
                for c in range(D):
                    acc[0][c] += Fraction(float(x[f, y, xx, c]))
                acc[1] += 1
    assert got.shape == (nT * Hb * Wb, D)
    for j, (s, n) in sums.items():
        assert n == (64 if (F % 2 and j < Hb * Wb) else 128)
        for c in range(D):
            assert got[j, c] == float(s[c] / n)  # exactly the correctly rounded mean


def test_pool_constant_blocks():
    F, Y, X, D = 4, 16, 24, 5
    rng = np.random.default_rng(0)
    consts = rng.integers(-50, 50, size=(2, 2, 3, D)) / 8.0
    x = np.zeros((F, Y, X, D))
    for f in range(F):
        for yb in range(2):
            for xb in range(3):
                x[f, yb * 8:(yb + 1) * 8, xb * 8:(xb + 1) * 8] = consts[f // 2, yb, xb]
    got = orc.pool_blocks(x).reshape(2, 2, 3, D)
    assert np.array_equal(got, consts)


def test_pool_rejects_inexact_sums():
    x = np.zeros((2, 8, 8, 1))
    x[0, 0, 0, 0] = 2.0 ** 40
    x[0, 0, 1, 0] = 2.0 ** -10
    with pytest.raises(ValueError):
        orc.pool_blocks(x)


# ----------------------------------------------------------------------------- scores
def test_scores_match_exact_dot_products():
    d = 16
    qp = _bf16_array((5, d), seed=3) / 128
    kp = _bf16_array((7, d), seed=4) / 128
    s = orc.block_scores(qp, kp)
    for i in range(5):
        for j in range(7):
            exact = sum(Fraction(float(a)) * Fraction(float(b)) for a, b in zip(qp[i], kp[j]))
            assert abs(s[i, j] * math.sqrt(d) - float(exact)) <= 1e-14 * (1 + abs(float(exact)))
    # transposed operands would break the shape and the values
    assert s.shape == (5, 7)


def test_scores_scale_is_one_over_sqrt_d():
    qp = np.ones((1, 64))
    kp = np.full((1, 64), 0.5)
    assert orc.block_scores(qp, kp)[0, 0] == 32.0 / 8.0


# ----------------------------------------------------------------------------- masks and K
def test_window_counts_hand_values():
    # 1536x2688 -> 96x168 tokens -> 12x21 blocks; 72x72-token window = 9x9 blocks
    Hb, Wb, w = 12, 21, 9
    corner_t = orc.allowed_blocks(0, 0, 0, 1, Hb, Wb, w, orc.WINDOW_TRUNCATE).sum()
    corner_p = orc.allowed_blocks(0, 0, 0, 1, Hb, Wb, w, orc.WINDOW_PRESERVE).sum()
    inner_t = orc.allowed_blocks(0, 6, 10, 1, Hb, Wb, w, orc.WINDOW_TRUNCATE).sum()
    edge_t = orc.allowed_blocks(0, 0, 10, 1, Hb, Wb, w, orc.WINDOW_TRUNCATE).sum()
    assert (corner_t, corner_p, inner_t, edge_t) == (25, 81, 81, 45)
    # three temporal blocks (2 query + 4 cached frames), causal from the newest
    assert orc.allowed_blocks(2, 0, 0, 3, Hb, Wb, w, orc.WINDOW_TRUNCATE).sum() == 75
    assert orc.allowed_blocks(2, 0, 0, 3, Hb, Wb, w, orc.WINDOW_PRESERVE).sum() == 243
    # preserve window is always w x w and contains the query block
    for y in range(Hb):
        for x in range(Wb):
            m = orc.allowed_blocks(0, y, x, 1, Hb, Wb, w, orc.WINDOW_PRESERVE).reshape(Hb, Wb)
            assert m.sum() == 81 and m[y, x]
            ys, xs = np.nonzero(m)
            assert ys.max() - ys.min() == 8 and xs.max() - xs.min() == 8


def test_window_truncate_equals_preserve_inside():
    Hb, Wb, w = 12, 21, 9
    for y in range(4, Hb - 4):
        for x in range(4, Wb - 4):
            a = orc.allowed_blocks(1, y, x, 2, Hb, Wb, w, orc.WINDOW_TRUNCATE)
            b = orc.allowed_blocks(1, y, x, 2, Hb, Wb, w, orc.WINDOW_PRESERVE)
            assert np.array_equal(a, b)


def test_window_larger_than_grid_is_no_window():
    Hb, Wb = 3, 5
    for mode in (orc.WINDOW_TRUNCATE, orc.WINDOW_PRESERVE):
        for y in range(Hb):
            for x in range(Wb):
                a = orc.allowed_blocks(1, y, x, 3, Hb, Wb, 11, mode)
                b = orc.allowed_blocks(1, y, x, 3, Hb, Wb, 0, mode)
                assert np.array_equal(a, b)


def test_causal_mask_is_block_level():
    m = orc.allowed_blocks(1, 0, 0, 3, 2, 2).reshape(3, 4)
    assert m[0].all() and m[1].all() and not m[2].any()


def test_k_rule_hand_values():
    # 768x1408 chunk: 3 temporal blocks x 66 = 198 candidates, 13.6% -> 27
    assert orc.top_k_count(198, density=0.136) == 27
    # 1536x2688 preserve: 3 x 81 = 243 candidates -> 34
    assert orc.top_k_count(243, density=0.136) == 34
    # whole clip: first and last temporal block (66 and 858 candidates)
    assert [orc.top_k_count(66, density=r) for r in (0.05, 0.136, 0.30)] == [4, 9, 20]
    assert [orc.top_k_count(858, density=r) for r in (0.05, 0.136, 0.30)] == [43, 117, 258]
    assert orc.top_k_count(4, top_k=2) == 2 and orc.top_k_count(1, top_k=2) == 1
    assert orc.top_k_count(3, density=0.01) == 1


# ----------------------------------------------------------------------------- top-K
def test_topk_golden_near_ties():
    fx = json.load(open(os.path.join(GOLDEN, "topk_near_ties.json")))
    for c in fx["cases"]:
        s = np.array(c["scores"])
        got = orc.select_row(s, np.ones(len(s), bool), c["K"], fx["eps"])
        assert got.tolist() == c["expect"], c["why"]


def test_topk_matches_brute_force_sort():
    rng = np.random.default_rng(7)
    for trial in range(300):
        C = int(rng.integers(1, 40))
        # well-separated scores (gaps > 2*eps): the tie rule reduces to plain top-K
        s = rng.permutation(C) * 1e-3 + rng.normal() * 0.1
        allowed = rng.random(C) < 0.7
        if not allowed.any():
            allowed[rng.integers(C)] = True
        K = int(rng.integers(1, allowed.sum() + 1))
        ranked = sorted((j for j in range(C) if allowed[j]), key=lambda j: (-s[j], j))
        assert orc.select_row(s, allowed, K).tolist() == sorted(ranked[:K])


def test_topk_k1_is_lowest_argmax():
    s = np.array([0.1, 0.9, 0.3, 0.9, 0.9])
    assert orc.select_row(s, np.ones(5, bool), 1).tolist() == [1]
    allowed = np.array([1, 0, 1, 1, 1], bool)
    assert orc.select_row(s, allowed, 1).tolist() == [3]


# ----------------------------------------------------------------------------- whole path
def _expand_blocks(vecs, frames, Y, X):
    """Token grid whose 2x8x8 blocks are constant, block vectors in (t, x) order."""
    D = len(vecs[0])
    a = np.zeros((frames, Y, X, D))
    Wb = X // 8
    for j, vec in enumerate(vecs):
        t, xb = divmod(j, Wb)
        a[2 * t:2 * t + 2, :, xb * 8:(xb + 1) * 8] = vec
    return a


def test_pipeline_golden_hand_case():
    fx = json.load(open(os.path.join(GOLDEN, "pipeline_hand.json")))
    g = fx["geometry"]
    q = _expand_blocks(fx["q_blocks"], g["q_frames"], g["Y"], g["X"])
    k = _expand_blocks(fx["k_blocks"], g["kv_frames"], g["Y"], g["X"])
    v = _expand_blocks(fx["v_blocks"], g["kv_frames"], g["Y"], g["X"])
    for c in fx["cases"]:
        r = orc.lcsa_head(q, k, v, top_k=c["top_k"])
        assert [s.tolist() for s in r["sel"]] == c["expect"], c["why"]
        assert r["C"].tolist() == [4, 4]
        if c["top_k"] == 3:
            e = math.exp(math.sqrt(2))
            v0, v1, v2 = (np.array(fx["v_blocks"][i], float) for i in range(3))
            o0 = (e * (v0 + v2) + v1) / (2 * e + 1)
            o1 = (v0 + e * (v1 + v2)) / (2 * e + 1)
            lse = math.log(128 * (2 * e + 1))
            assert np.allclose(r["O"][:, :, 0:8], o0, atol=1e-14)
            assert np.allclose(r["O"][:, :, 8:16], o1, atol=1e-14)
            assert np.allclose(r["LSE"], lse, atol=1e-13)


def _dense_block_causal_sdpa(q, k, v):
    """Dense attention with a boolean block-causal mask, via torch in float64."""
    Tq, Y, X, D = q.shape
    F = k.shape[0]
    nQT, nKT = (Tq + 1) // 2, (F + 1) // 2
    qt = np.repeat([_tblk(f, Tq) + nKT - nQT for f in range(Tq)], Y * X)
    kt = np.repeat([_tblk(f, F) for f in range(F)], Y * X)
    mask = torch.from_numpy(kt[None, :] <= qt[:, None])
    o = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q.reshape(1, -1, D)), torch.from_numpy(k.reshape(1, -1, D)),
        torch.from_numpy(v.reshape(1, -1, D)), attn_mask=mask)
    return o.numpy().reshape(q.shape)


@pytest.mark.parametrize("Tq,F", [(2, 6), (4, 4), (2, 5)])
def test_full_density_equals_dense_block_causal(Tq, F):
    Y, X, D = 16, 16, 8
    q = _bf16_array((Tq, Y, X, D), seed=20 + F)
    k = _bf16_array((F, Y, X, D), seed=30 + F)
    v = _bf16_array((F, Y, X, D), seed=40 + F)
    r = orc.lcsa_head(q, k, v, density=1.0)
    assert all(len(s) == c for s, c in zip(r["sel"], r["C"]))
    ref = _dense_block_causal_sdpa(q, k, v)
    assert np.max(np.abs(r["O"] - ref)) < 1e-12


def test_rows_sum_to_one():
    Y, X, D = 16, 24, 8
    q = _bf16_array((2, Y, X, D), seed=50)
    k = _bf16_array((6, Y, X, D), seed=51)
    r = orc.lcsa_head(q, k, np.ones((6, Y, X, D)), density=0.3)
    assert np.max(np.abs(r["O"] - 1.0)) < 1e-13
    # each row's LSE is the log of the sum of its unnormalised weights
    sel0 = r["sel"][0]
    keys = orc.gather_blocks(k, sel0)
    logits = keys @ q[0, 0, 0] / math.sqrt(D)
    assert abs(r["LSE"][0, 0, 0] - math.log(np.exp(logits).sum())) < 1e-12


def test_single_block_is_textbook_attention():
    Y, X, D = 8, 8, 16
    q = _bf16_array((2, Y, X, D), seed=60)
    k = _bf16_array((4, Y, X, D), seed=61)
    v = _bf16_array((4, Y, X, D), seed=62)
    r = orc.lcsa_head(q, k, v, top_k=1)
    (j,) = r["sel"][0]
    t = int(j)
    kb = k[2 * t:2 * t + 2].reshape(-1, D)
    vb = v[2 * t:2 * t + 2].reshape(-1, D)
    qq = q.reshape(-1, D)
    w = np.exp(qq @ kb.T / 4.0)
    expect = (w / w.sum(axis=1, keepdims=True)) @ vb
    assert np.max(np.abs(r["O"].reshape(-1, D) - expect)) < 1e-13


def test_block_order_does_not_change_output():
    Y, X, D = 16, 16, 8
    q = _bf16_array((2, Y, X, D), seed=70)
    k = _bf16_array((6, Y, X, D), seed=71)
    v = _bf16_array((6, Y, X, D), seed=72)
    r = orc.lcsa_head(q, k, v, density=0.5)
    perm = [s[::-1].copy() for s in r["sel"]]
    O2, L2 = orc.attend_head(q, k, v, perm)
    assert np.max(np.abs(O2 - r["O"])) < 1e-13 and np.max(np.abs(L2 - r["LSE"])) < 1e-12


def test_window_at_least_grid_selects_like_no_window():
    Y, X, D = 16, 24, 8
    q = _bf16_array((2, Y, X, D), seed=80)
    k = _bf16_array((4, Y, X, D), seed=81)
    v = _bf16_array((4, Y, X, D), seed=82)
    a = orc.lcsa_head(q, k, v, density=0.4)
    for mode in (orc.WINDOW_TRUNCATE, orc.WINDOW_PRESERVE):
        b = orc.lcsa_head(q, k, v, density=0.4, window=7, mode=mode)
        assert all(np.array_equal(x, y) for x, y in zip(a["sel"], b["sel"]))


def test_selection_stays_in_window_and_is_causal():
    Y, X, D = 48, 56, 8
    q = _bf16_array((2, Y, X, D), seed=90)
    k = _bf16_array((4, Y, X, D), seed=91)
    v = _bf16_array((4, Y, X, D), seed=92)
    r = orc.lcsa_head(q, k, v, density=0.3, window=3, mode=orc.WINDOW_TRUNCATE)
    Hb, Wb = 6, 7
    for i, s in enumerate(r["sel"]):
        yq, xq = divmod(i % (Hb * Wb), Wb)
        for j in s:
            t, rr = divmod(int(j), Hb * Wb)
            yk, xk = divmod(rr, Wb)
            assert t <= 1 and abs(yk - yq) <= 1 and abs(xk - xq) <= 1


# ----------------------------------------------------------------------------- KV cache
def test_kv_append_concatenates_and_evicts():
    a = np.arange(5)[:, None] * np.ones((5, 3))
    b = np.arange(5, 7)[:, None] * np.ones((2, 3))
    c = orc.kv_append(a, b, cap_frames=6)
    assert c[:, 0].tolist() == [1, 2, 3, 4, 5, 6]
    assert orc.kv_append(None, b, 8)[:, 0].tolist() == [5, 6]
    assert orc.kv_append(a, b, 8)[:, 0].tolist() == list(range(7))
