"""fp64 CPU oracle for FlashVSR's locality-constrained block-sparse causal attention.

TEST INFRASTRUCTURE. Only the tests, ``__graft_entry__.smoke()`` and the CPU
baseline / reference legs of ``bench.py`` may import or run this module. The
library never calls it and shares no code with it: the CUDA path and this file
meet only in the seeded input generators of ``lcsa_inputs``.

What it computes (FlashVSR, "Towards Real-time Diffusion-Based Streaming Video
Super-Resolution"; the fmread summary of the paper, section 2.2 "stage 2:
block-sparse causal attention adaptation", section 2.2 "stage 3" for the KV
cache, section 2.3 "locality-constrained sparse attention"):

1. Q and K are cut into non-overlapping 2x8x8 (t, y, x) token blocks and each
   block is mean-pooled into one feature vector (``pool_blocks``).
2. A coarse block-to-block map is formed from the pooled features
   (``block_scores``), restricted by the causal mask over time and, at
   inference, by a spatial locality window with a boundary-truncate or a
   boundary-preserve rule (``allowed_blocks``).
3. Only the top-K key blocks per query block are kept (``select_row``).
4. Full softmax attention runs over the tokens of the kept blocks
   (``attend_rows``); its gradients for training follow by the chain rule
   with the selection held fixed (``attend_rows_backward``).
5. The streaming KV cache appends each chunk and drops the oldest frames
   (``kv_append``).

Everything is float64, from the bf16 input bits widened exactly. Readings of
points the pages leave open (block alignment in time, block-level causality,
the window rules, the K rule and the tie rule) are stated on each function.

Pins (checked in ``tests/test_oracle_pins.py`` against things other than this
file): exact rational means, brute-force top-K, hand-derived golden cases,
full-density equality with masked dense attention from torch, unit row sums,
the single-block textbook case, window invariants; for the gradients: central
finite differences, torch autograd of masked dense attention, and the closed
forms sum_t dk_t = 0, sum_t dv_t = sum_r do_r, dq = dk = 0 for equal values. Parity with the authors'
own implementation is unpinned: the pages print no numeric example of it.
"""
from __future__ import annotations

import math
from typing import List, Sequence, Tuple

import numpy as np

BLOCK_T, BLOCK_Y, BLOCK_X = 2, 8, 8
WINDOW_TRUNCATE, WINDOW_PRESERVE = 0, 1
WINDOW_TRUNCATE_TOKENS = 2   # token-level window, clipped at the frame edge
WINDOW_PRESERVE_TOKENS = 3   # token-level window, shifted inward at the edge
TIE_EPS = 1e-5

# Largest exponent spread (in binades) among the non-zero terms of one block sum
# for which a float64 sum of at most 128 bf16 values is exact in any order.
EXACT_SUM_SPAN = 38


# --------------------------------------------------------------------------- #
# Block geometry (section 2.2, stage 2: "blocks of size 2x8x8")
# --------------------------------------------------------------------------- #
def temporal_blocks(F: int) -> List[List[int]]:
    """Frame indices of each temporal block of an F-frame sequence, oldest first.

    Reading: blocks of two frames are counted backwards from the newest frame,
    aligned with the streaming chunk; an odd F leaves the OLDEST block with a
    single frame. (The pages give only the block size.)
    """
    n = (F + 1) // 2
    off = F - 2 * n  # 0, or -1 when F is odd
    return [[f for f in (off + 2 * t, off + 2 * t + 1) if f >= 0] for t in range(n)]


def block_grid(F: int, Y: int, X: int) -> Tuple[int, int, int]:
    """(temporal blocks, block rows, block columns) of an F x Y x X token grid."""
    if Y % BLOCK_Y or X % BLOCK_X:
        raise ValueError("token grid must be a multiple of 8 in y and x")
    return (F + 1) // 2, Y // BLOCK_Y, X // BLOCK_X


def block_token_view(x: np.ndarray, frames: Sequence[int], yb: int, xb: int) -> np.ndarray:
    """Tokens of one block as ``[n_tokens][D]`` in (t, y, x) order."""
    sub = x[list(frames), yb * BLOCK_Y:(yb + 1) * BLOCK_Y, xb * BLOCK_X:(xb + 1) * BLOCK_X, :]
    return sub.reshape(-1, x.shape[-1])


# --------------------------------------------------------------------------- #
# 1. Pooling (section 2.2, stage 2: "average pooling yields block-level features")
# --------------------------------------------------------------------------- #
def _assert_exact_sums(blocks: np.ndarray) -> None:
    """Check that every per-channel block sum is exact in float64.

    ``blocks`` is ``[nBlk][n_tokens][D]`` of widened bf16 values. Each value is
    an 8-bit significand times a power of two, so a sum of at most 128 of them
    is exact (hence independent of summation order) when the exponents of its
    non-zero terms span at most 38 binades: all terms and partial sums are then
    integer multiples of the smallest term's unit and stay below 2**53 of it.
    """
    a = np.abs(blocks)
    _, e = np.frexp(a)
    nz = a > 0
    emax = np.where(nz, e, -10**6).max(axis=1)
    emin = np.where(nz, e, 10**6).min(axis=1)
    span = np.where(nz.any(axis=1), emax - emin, 0)
    if int(span.max(initial=0)) > EXACT_SUM_SPAN:
        raise ValueError("block sum not exact in float64 (exponent span %d)" % int(span.max()))


def pool_blocks(x: np.ndarray) -> np.ndarray:
    """Mean of each 2x8x8 block of ``x`` (float64 ``[F][Y][X][D]``).

    Returns ``[nT*Hb*Wb][D]``, block id = t_blk*Hb*Wb + y_blk*Wb + x_blk with
    t_blk oldest first. A one-frame block averages its 64 tokens.
    """
    F, Y, X, D = x.shape
    nT, Hb, Wb = block_grid(F, Y, X)
    out = np.empty((nT * Hb * Wb, D))
    for t, frames in enumerate(temporal_blocks(F)):
        # [nf][Hb][8][Wb][8][D] -> [Hb][Wb][nf*8*8][D]
        sub = x[frames].reshape(len(frames), Hb, BLOCK_Y, Wb, BLOCK_X, D)
        tok = sub.transpose(1, 3, 0, 2, 4, 5).reshape(Hb * Wb, -1, D)
        _assert_exact_sums(tok)
        out[t * Hb * Wb:(t + 1) * Hb * Wb] = tok.sum(axis=1) / tok.shape[1]
    return out


# --------------------------------------------------------------------------- #
# 2. Coarse block map and masks (section 2.2 stage 2 causal masking and the
#    "coarse block-to-block attention map"; section 2.3 locality window)
# --------------------------------------------------------------------------- #
def block_scores(qp: np.ndarray, kp: np.ndarray) -> np.ndarray:
    """Scaled block logits s_ij = (qbar_i . kbar_j) / sqrt(d).

    The dot product is summed channel by channel in order c = 0..d-1, each
    product rounded before it is added (no fused multiply-add), then divided by
    the correctly rounded sqrt(d). Fixing this order makes the scores a
    definite float64 value, so block selections can be compared bit for bit.
    """
    d = qp.shape[1]
    s = np.zeros((qp.shape[0], kp.shape[0]))
    for c in range(d):
        s = s + np.multiply.outer(qp[:, c], kp[:, c])
    return s / math.sqrt(d)


def window_range(i: int, n: int, window: int, mode: int) -> Tuple[int, int]:
    """Half-open range of block coordinates along one axis seen from block i.

    Reading of the two rules the pages name: the window is ``window`` blocks
    wide, centred on the query block (radius r = window // 2).
      truncate: [i-r, i+r] clipped to the frame, so it shrinks at the edge;
      preserve: shifted inward at the edge so it always spans ``window``
                blocks (start = max(0, min(i-r, n-window))).
    A window at least as large as the frame covers the whole axis.
    """
    r = window // 2
    if mode == WINDOW_TRUNCATE:
        return max(0, i - r), min(n, i + r + 1)
    if mode == WINDOW_PRESERVE:
        start = max(0, min(i - r, n - window))
        return start, min(n, start + window)
    raise ValueError("unknown window mode")


def token_window_range(p: int, n: int, window: int, mode: int) -> Tuple[int, int]:
    """Half-open range of token coordinates along one axis seen from query token p.

    Token-level reading of "each query's attention is limited to a local
    neighbourhood" (e.g. 1152 px = 72 tokens): the window is ``window`` tokens
    wide with the query at offset window // 2 (window // 2 tokens before it,
    the rest after), truncated at the frame edge or, with preserve, shifted
    inward so it keeps its width (start = max(0, min(p - window//2, n - window))).
    """
    s = p - window // 2
    if mode == WINDOW_TRUNCATE_TOKENS:
        return max(0, s), min(n, s + window)
    if mode == WINDOW_PRESERVE_TOKENS:
        st = max(0, min(s, n - window))
        return st, min(n, st + window)
    raise ValueError("unknown token window mode")


def token_block_range(i: int, n_tokens: int, window: int, mode: int) -> Tuple[int, int]:
    """Half-open range of block coordinates along one axis holding at least one
    token that some token of block i sees (the union of its tokens' windows;
    both window ends move monotonically with the query token)."""
    lo = token_window_range(BLOCK_Y * i, n_tokens, window, mode)[0]
    hi = token_window_range(BLOCK_Y * i + BLOCK_Y - 1, n_tokens, window, mode)[1]
    return lo // BLOCK_Y, (hi - 1) // BLOCK_Y + 1


def allowed_blocks(tq: int, yq: int, xq: int, nKT: int, Hb: int, Wb: int,
                   window: int = 0, mode: int = WINDOW_TRUNCATE) -> np.ndarray:
    """Boolean mask over the nKT*Hb*Wb key blocks for query block (tq, yq, xq).

    ``tq`` is the query block's temporal index in the key timeline. Causal
    reading: block-level, t_key <= t_query, so the two frames of one block (one
    streaming chunk) see each other fully. The window is spatial only and
    applies at every past time step.
    """
    m = np.zeros((nKT, Hb, Wb), dtype=bool)
    if window > 0 and mode in (WINDOW_TRUNCATE_TOKENS, WINDOW_PRESERVE_TOKENS):
        y0, y1 = token_block_range(yq, Hb * BLOCK_Y, window, mode)
        x0, x1 = token_block_range(xq, Wb * BLOCK_X, window, mode)
        m[:tq + 1, y0:y1, x0:x1] = True
        return m.reshape(-1)
    y0, y1 = (0, Hb) if window <= 0 else window_range(yq, Hb, window, mode)
    x0, x1 = (0, Wb) if window <= 0 else window_range(xq, Wb, window, mode)
    m[:tq + 1, y0:y1, x0:x1] = True
    return m.reshape(-1)


# --------------------------------------------------------------------------- #
# 3. Top-K (section 2.2, stage 2: keep only the most relevant top-K block pairs)
# --------------------------------------------------------------------------- #
def top_k_count(C: int, top_k: int = 0, density: float = 0.0) -> int:
    """K_i for a row with C allowed key blocks.

    Fixed K: min(C, top_k). Density rho: K = min(C, max(1, ceil(rho*C))) with
    rho*C a float64 product, i.e. rho is read as the kept fraction of the
    allowed (causal, in-window) pairs of each row.
    """
    if top_k > 0:
        return min(C, top_k)
    return min(C, max(1, math.ceil(density * C)))


def select_row(s_row: np.ndarray, allowed: np.ndarray, K: int,
               eps: float = TIE_EPS) -> np.ndarray:
    """Indices (ascending) of the K kept key blocks of one query block.

    tau is the K-th largest allowed score, hi = tau + eps and lo = tau - eps
    (float64). Every allowed block with s > hi is kept; the remaining places go
    to the lowest-index blocks with lo <= s <= hi, so near-ties within eps of
    the K-th score are resolved by block index.
    """
    idx = np.nonzero(allowed)[0]
    vals = s_row[idx]
    tau = np.sort(vals)[::-1][K - 1]
    hi, lo = tau + eps, tau - eps
    above = vals > hi
    band = (vals >= lo) & (vals <= hi)
    need = K - int(above.sum())
    return np.sort(np.concatenate([idx[above], idx[band][:need]]))


# --------------------------------------------------------------------------- #
# 4. Attention over the kept blocks (section 2.2, stage 2: "full attention
#    inside the selected regions")
# --------------------------------------------------------------------------- #
def attend_rows(q: np.ndarray, k: np.ndarray, v: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    """Softmax attention of rows ``q`` [n][d] over keys ``k``/values ``v`` [m][d].

    O = softmax(q k^T / sqrt(d)) v and LSE = log sum exp(q k^T / sqrt(d)), the
    textbook definition in float64.
    """
    s = (q @ k.T) / math.sqrt(q.shape[1])
    mx = s.max(axis=1, keepdims=True)
    e = np.exp(s - mx)
    l = e.sum(axis=1, keepdims=True)
    return (e / l) @ v, mx[:, 0] + np.log(l[:, 0])


def attend_rows_masked(q: np.ndarray, k: np.ndarray, v: np.ndarray,
                       mask: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    """``attend_rows`` with a boolean visibility mask [n][m]: masked keys get
    zero weight. A row that sees no key at all has O = 0 and LSE = -inf."""
    s = (q @ k.T) / math.sqrt(q.shape[1])
    s = np.where(mask, s, -np.inf)
    mx = s.max(axis=1, keepdims=True)
    empty = ~np.isfinite(mx[:, 0])
    mx = np.where(np.isfinite(mx), mx, 0.0)
    e = np.where(mask, np.exp(s - mx), 0.0)
    l = e.sum(axis=1, keepdims=True)
    o = (e / np.where(l > 0, l, 1.0)) @ v
    lse = mx[:, 0] + np.log(np.where(l[:, 0] > 0, l[:, 0], 1.0))
    o[empty] = 0.0
    lse[empty] = -np.inf
    return o, lse


def token_yx(F: int, Y: int, X: int, ids: Sequence[int]) -> Tuple[np.ndarray, np.ndarray]:
    """(y, x) token coordinates of the tokens of the given blocks, in the order
    ``gather_blocks`` concatenates them."""
    flat = block_token_index(F, Y, X, ids) % (Y * X)
    return flat // X, flat % X


def gather_blocks(x: np.ndarray, ids: Sequence[int]) -> np.ndarray:
    """Tokens of the given key blocks of ``x`` [F][Y][X][D], concatenated."""
    F, Y, X, _ = x.shape
    _, Hb, Wb = block_grid(F, Y, X)
    tb = temporal_blocks(F)
    parts = []
    for j in ids:
        t, r = divmod(int(j), Hb * Wb)
        yb, xb = divmod(r, Wb)
        parts.append(block_token_view(x, tb[t], yb, xb))
    return np.concatenate(parts, axis=0)


# --------------------------------------------------------------------------- #
# 4b. Gradients of the attention over the kept blocks. The pages train stage 2
#     (and stage 3) with the block-sparse causal mask (section 2.2, stage 2:
#     "trained with the flow-matching loss"), so the attention needs its
#     backward pass. The selection is a constant mask: the top-K of pooled
#     scores is piecewise constant, its derivative is zero almost everywhere.
# --------------------------------------------------------------------------- #
def attend_rows_backward(q: np.ndarray, k: np.ndarray, v: np.ndarray,
                         do: np.ndarray) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """Gradients of O = softmax(q k^T / sqrt(d)) v with respect to q, k, v for
    the output gradient ``do``, by the chain rule through the row softmax:

        P = softmax(S), S = q k^T / sqrt(d), O = P v
        dV = P^T dO,  dP = dO v^T,  delta_r = sum_d dO_rd O_rd (= sum_t P_rt dP_rt)
        dS = P * (dP - delta),  dq = dS k / sqrt(d),  dk = dS^T q / sqrt(d)
    """
    scale = 1.0 / math.sqrt(q.shape[1])
    s = (q @ k.T) * scale
    e = np.exp(s - s.max(axis=1, keepdims=True))
    p = e / e.sum(axis=1, keepdims=True)
    o = p @ v
    dv = p.T @ do
    dp = do @ v.T
    delta = (do * o).sum(axis=1, keepdims=True)
    ds = p * (dp - delta)
    return (ds @ k) * scale, (ds.T @ q) * scale, dv


def block_token_index(F: int, Y: int, X: int, ids: Sequence[int]) -> np.ndarray:
    """Flat indices into [F][Y][X] of the tokens of the given blocks, in the
    order ``gather_blocks`` concatenates them."""
    _, Hb, Wb = block_grid(F, Y, X)
    tb = temporal_blocks(F)
    flat = np.arange(F * Y * X).reshape(F, Y, X)
    parts = []
    for j in ids:
        t, r = divmod(int(j), Hb * Wb)
        yb, xb = divmod(r, Wb)
        parts.append(block_token_view(flat[..., None], tb[t], yb, xb)[:, 0])
    return np.concatenate(parts)


def attend_head_backward(q: np.ndarray, k: np.ndarray, v: np.ndarray, sel: Sequence[np.ndarray],
                         do: np.ndarray):
    """dq, dk, dv of one (stream, head): ``q``/``do`` [Tq][Y][X][D], ``k``/``v``
    [F][Y][X][D], ``sel`` the kept key blocks of every query block. Each query
    block's gradients come from ``attend_rows_backward`` over its kept tokens;
    the key and value gradients of all query blocks are summed per token."""
    Tq, Y, X, D = q.shape
    F = k.shape[0]
    nQT, Hb, Wb = block_grid(Tq, Y, X)
    dq = np.zeros(q.shape)
    dk = np.zeros(k.shape).reshape(-1, D)
    dv = np.zeros(v.shape).reshape(-1, D)
    kf, vf = k.reshape(-1, D), v.reshape(-1, D)
    for i in range(nQT * Hb * Wb):
        qidx = block_token_index(Tq, Y, X, [i])
        kidx = block_token_index(F, Y, X, sel[i])
        gq, gk, gv = attend_rows_backward(q.reshape(-1, D)[qidx], kf[kidx], vf[kidx], do.reshape(-1, D)[qidx])
        dq.reshape(-1, D)[qidx] = gq
        np.add.at(dk, kidx, gk)
        np.add.at(dv, kidx, gv)
    return dq, dk.reshape(k.shape), dv.reshape(v.shape)


# --------------------------------------------------------------------------- #
# 4c. Dense attention confined to one segment (section 2.2, stage 1: joint
#     video-image training with a block-diagonal segment mask; an image is a
#     one-frame video). Within a segment every query token sees every key
#     token of the segment, past or future; nothing crosses segments.
# --------------------------------------------------------------------------- #
def segment_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    """O [F_q][Y][X][D] and LSE [F_q][Y][X] of the segment's query tokens over
    all of its key tokens (``attend_rows`` on the flattened tokens)."""
    D = q.shape[-1]
    o, lse = attend_rows(q.reshape(-1, D), k.reshape(-1, D), v.reshape(-1, D))
    return o.reshape(q.shape), lse.reshape(q.shape[:3])


def segment_attention_backward(q: np.ndarray, k: np.ndarray, v: np.ndarray, do: np.ndarray):
    """dq, dk, dv of ``segment_attention`` (``attend_rows_backward`` on the
    flattened tokens)."""
    D = q.shape[-1]
    dq, dk, dv = attend_rows_backward(q.reshape(-1, D), k.reshape(-1, D), v.reshape(-1, D), do.reshape(-1, D))
    return dq.reshape(q.shape), dk.reshape(k.shape), dv.reshape(v.shape)


# --------------------------------------------------------------------------- #
# One (stream, head): pool -> scores -> masks -> top-K -> attention
# --------------------------------------------------------------------------- #
def select_head(qp: np.ndarray, kp: np.ndarray, q_frames: int, kv_frames: int, Y: int, X: int,
                top_k: int = 0, density: float = 0.0, window: int = 0,
                mode: int = WINDOW_TRUNCATE, eps: float = TIE_EPS):
    """Selections of every query block of one (stream, head).

    The queries are the last ``q_frames`` frames of the ``kv_frames``-frame key
    timeline, so query temporal block t sits at key temporal block
    nKT - nQT + t. Returns (list of index arrays, K_i array, C_i array).
    """
    nQT, Hb, Wb = block_grid(q_frames, Y, X)
    nKT, _, _ = block_grid(kv_frames, Y, X)
    if q_frames > kv_frames:
        raise ValueError("queries must be the newest frames of the key timeline")
    s = block_scores(qp, kp)
    sel, Ks, Cs = [], [], []
    for i in range(nQT * Hb * Wb):
        t, r = divmod(i, Hb * Wb)
        yq, xq = divmod(r, Wb)
        allowed = allowed_blocks(nKT - nQT + t, yq, xq, nKT, Hb, Wb, window, mode)
        C = int(allowed.sum())
        K = top_k_count(C, top_k, density)
        sel.append(select_row(s[i], allowed, K, eps))
        Ks.append(K)
        Cs.append(C)
    return sel, np.array(Ks), np.array(Cs)


def attend_head(q: np.ndarray, k: np.ndarray, v: np.ndarray, sel: Sequence[np.ndarray],
                rows: Sequence[int] | None = None, window: int = 0, mode: int = WINDOW_TRUNCATE):
    """Attention output of one (stream, head) for the given selections.

    ``q`` [Tq][Y][X][D], ``k``/``v`` [F][Y][X][D] float64. Returns O laid out
    like ``q`` and LSE ``[Tq][Y][X]``; with ``rows`` given, only those query
    blocks are computed (the others stay NaN).
    """
    Tq, Y, X, D = q.shape
    nQT, Hb, Wb = block_grid(Tq, Y, X)
    qtb = temporal_blocks(Tq)
    O = np.full(q.shape, np.nan)
    L = np.full(q.shape[:3], np.nan)
    for i in (range(nQT * Hb * Wb) if rows is None else rows):
        t, r = divmod(int(i), Hb * Wb)
        yb, xb = divmod(r, Wb)
        qi = block_token_view(q, qtb[t], yb, xb)
        if window > 0 and mode in (WINDOW_TRUNCATE_TOKENS, WINDOW_PRESERVE_TOKENS):
            # token-level window inside the kept blocks: key (yk, xk) is visible
            # to query (yq, xq) iff yk and xk lie in the query token's windows
            qy, qx = token_yx(Tq, Y, X, [i])
            ky, kx = token_yx(k.shape[0], Y, X, sel[i])
            vis = np.ones((qy.size, ky.size), dtype=bool)
            for a, (yy, xx) in enumerate(zip(qy, qx)):
                y0, y1 = token_window_range(int(yy), Y, window, mode)
                x0, x1 = token_window_range(int(xx), X, window, mode)
                vis[a] = (ky >= y0) & (ky < y1) & (kx >= x0) & (kx < x1)
            o, lse = attend_rows_masked(qi, gather_blocks(k, sel[i]), gather_blocks(v, sel[i]), vis)
        else:
            o, lse = attend_rows(qi, gather_blocks(k, sel[i]), gather_blocks(v, sel[i]))
        ys, xs = slice(yb * BLOCK_Y, (yb + 1) * BLOCK_Y), slice(xb * BLOCK_X, (xb + 1) * BLOCK_X)
        O[qtb[t], ys, xs, :] = o.reshape(len(qtb[t]), BLOCK_Y, BLOCK_X, D)
        L[qtb[t], ys, xs] = lse.reshape(len(qtb[t]), BLOCK_Y, BLOCK_X)
    return O, L


def lcsa_head(q: np.ndarray, k: np.ndarray, v: np.ndarray, top_k: int = 0,
              density: float = 0.0, window: int = 0, mode: int = WINDOW_TRUNCATE,
              eps: float = TIE_EPS, rows: Sequence[int] | None = None) -> dict:
    """The whole path for one (stream, head) on float64 arrays."""
    qp, kp = pool_blocks(q), pool_blocks(k)
    sel, Ks, Cs = select_head(qp, kp, q.shape[0], k.shape[0], q.shape[1], q.shape[2],
                              top_k, density, window, mode, eps)
    O, L = attend_head(q, k, v, sel, rows, window, mode)
    return {"q_pool": qp, "k_pool": kp, "sel": sel, "K": Ks, "C": Cs, "O": O, "LSE": L}


# --------------------------------------------------------------------------- #
# 5. Streaming KV cache (section 2.2, stage 3: temporal consistency through a
#    KV cache in later layers; section 3: 8-frame streaming chunks)
# --------------------------------------------------------------------------- #
def kv_append(frames: np.ndarray | None, new: np.ndarray, cap_frames: int) -> np.ndarray:
    """Cache after appending ``new`` [Tn][...] to ``frames`` [F][...]: the last
    ``cap_frames`` frames of their concatenation, oldest first."""
    cat = new if frames is None or len(frames) == 0 else np.concatenate([frames, new], axis=0)
    return cat[max(0, cat.shape[0] - cap_frames):]


def widen(t) -> np.ndarray:
    """bf16 torch tensor -> float64 numpy array (exact)."""
    return t.float().double().numpy() if hasattr(t, "float") else np.asarray(t, dtype=np.float64)
