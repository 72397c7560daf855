"""How several GPUs share one batch of streams.

Every (stream, head) pair is an independent unit of the attention path:
pooling, the coarse map, the top-K, the sparse attention and the KV cache of
one head of one video stream read nothing of any other pair (FlashVSR summary,
section 2.2 stage 2: the block map and the top-K are per head; stage 3: the KV
cache is per stream). So ranks split the units with no data-path exchange.

The units are numbered stream-major (stream 0's heads first) and rank r takes
the contiguous range [r*U/N, (r+1)*U/N) of the U = streams x heads units: when
the streams divide evenly over the ranks each rank gets whole streams, and
otherwise the remainder is split by heads. Unit counts of any two ranks differ
by at most one. Each rank runs its share as one call per stream range, with
the heads of that range (a [1][h1-h0] slice of the stream's tensors).
"""
from __future__ import annotations

from typing import List, Tuple

__all__ = ["rank_units", "rank_slices"]


def rank_units(n_streams: int, n_heads: int, world: int, rank: int) -> List[Tuple[int, int]]:
    """The (stream, head) units of `rank` among `world` ranks, in order."""
    if n_streams < 1 or n_heads < 1 or world < 1 or not 0 <= rank < world:
        raise ValueError("need n_streams, n_heads, world >= 1 and 0 <= rank < world")
    total = n_streams * n_heads
    lo = rank * total // world
    hi = (rank + 1) * total // world
    return [divmod(u, n_heads) for u in range(lo, hi)]


def rank_slices(n_streams: int, n_heads: int, world: int, rank: int) -> List[Tuple[int, int, int]]:
    """The same share as (stream, head_begin, head_end) ranges, one per stream
    the rank touches (at most ceil(streams/world) + 1 of them)."""
    out: List[Tuple[int, int, int]] = []
    for b, h in rank_units(n_streams, n_heads, world, rank):
        if out and out[-1][0] == b and out[-1][2] == h:
            out[-1] = (b, out[-1][1], h + 1)
        else:
            out.append((b, h, h + 1))
    return out
