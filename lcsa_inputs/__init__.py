"""Seeded synthetic inputs for locality-constrained block-sparse causal attention.

This module only draws random tensors and lays them out in the shapes of the
workloads. It holds none of the attention method's arithmetic (no pooling,
scoring, selection or softmax), so the CUDA path and the fp64 oracle can both
consume exactly the same bf16 bits without sharing any code of the method.

Every tensor is drawn with ``torch.Generator(device="cpu").manual_seed(seed)``
as fp32 ``randn``, then given the workload's structure, then rounded once to
bf16. Layouts are ``[H][F][Y][X][D]`` per stream (D contiguous): heads, latent
frames, token rows, token columns, channels. One token covers 16x16 output
pixels, so a 768x1408 video is a 48x88 token grid per latent frame.

Workloads (FlashVSR, "Towards Real-time Diffusion-Based Streaming Video Super
Resolution", section 2 "three-stage distillation", stage 2 block-sparse causal
attention; section 3 locality-constrained attention; section 3 efficiency
analysis for the 768x1408 and 1536x2688 sizes):

* ``tiny``        1 head, d=64, 2x16x16 tokens, fixed K=2, no window.
* ``chunk``       12 heads, d=128, 48x88 tokens per frame, a 2-frame query
                  chunk against a cache of the chunk plus 4 past frames,
                  3D RoPE on Q and K, 13.6% of causal block pairs kept.
* ``clip``        the whole 101-frame clip: 26 latent frames, block-causal,
                  Q/K with a smooth low-frequency spatial field added.
* ``multistream`` 4 streams, 2-frame chunks, caches holding 4, 5 or 6 past
                  frames (ragged, from the seed), capacity 6 past frames.
* ``uhr``         96x168 tokens per frame (1536x2688), 2+4 frames, a 9x9
                  block (72x72 token, 1152x1152 pixel) locality window.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace
from typing import List, Tuple

import torch

__all__ = ["Workload", "WORKLOADS", "workload", "make_inputs", "small_variant"]

WINDOW_TRUNCATE = 0
WINDOW_PRESERVE = 1
WINDOW_TRUNCATE_TOKENS = 2
WINDOW_PRESERVE_TOKENS = 3


@dataclass(frozen=True)
class Workload:
    """Shape and sampling recipe of one synthetic workload.

    A stream's timeline holds ``kv_past[b]`` past latent frames followed by the
    ``q_frames`` frames of the current chunk; the queries are the current
    chunk, the keys/values are the whole timeline (at most ``cap_frames``).
    """

    name: str
    B: int
    H: int
    D: int
    Y: int
    X: int
    q_frames: int
    kv_past: Tuple[int, ...]
    cap_frames: int
    top_k: int = 0
    density: float = 0.0
    window: int = 0
    window_mode: int = WINDOW_TRUNCATE
    seed: int = 0
    structure: str = "iid"  # "iid" | "rope" | "field"

    @property
    def kv_frames(self) -> Tuple[int, ...]:
        return tuple(p + self.q_frames for p in self.kv_past)

    @property
    def Hb(self) -> int:
        return self.Y // 8

    @property
    def Wb(self) -> int:
        return self.X // 8


def _ms_past(seed: int) -> Tuple[int, ...]:
    # 4 streams whose past lengths cover 4, 5 and 6 frames, order from the seed.
    g = torch.Generator(device="cpu").manual_seed(seed)
    extra = int(torch.randint(4, 7, (1,), generator=g).item())
    vals = torch.tensor([4, 5, 6, extra])
    perm = torch.randperm(4, generator=g)
    return tuple(int(v) for v in vals[perm])


WORKLOADS = {
    "tiny": Workload("tiny", B=1, H=1, D=64, Y=16, X=16, q_frames=2, kv_past=(0,),
                     cap_frames=2, top_k=2, seed=1),
    "chunk": Workload("chunk", B=1, H=12, D=128, Y=48, X=88, q_frames=2, kv_past=(4,),
                      cap_frames=6, density=0.136, seed=2, structure="rope"),
    "clip_5": Workload("clip_5", B=1, H=12, D=128, Y=48, X=88, q_frames=26, kv_past=(0,),
                       cap_frames=26, density=0.05, seed=3, structure="field"),
    "clip": Workload("clip", B=1, H=12, D=128, Y=48, X=88, q_frames=26, kv_past=(0,),
                     cap_frames=26, density=0.136, seed=3, structure="field"),
    "clip_30": Workload("clip_30", B=1, H=12, D=128, Y=48, X=88, q_frames=26, kv_past=(0,),
                        cap_frames=26, density=0.30, seed=3, structure="field"),
    "multistream": Workload("multistream", B=4, H=12, D=128, Y=48, X=88, q_frames=2,
                            kv_past=_ms_past(4), cap_frames=8, density=0.136, seed=4),
    "uhr_truncate": Workload("uhr_truncate", B=1, H=12, D=128, Y=96, X=168, q_frames=2,
                             kv_past=(4,), cap_frames=6, density=0.136, window=9,
                             window_mode=WINDOW_TRUNCATE, seed=5),
    "uhr_preserve": Workload("uhr_preserve", B=1, H=12, D=128, Y=96, X=168, q_frames=2,
                             kv_past=(4,), cap_frames=6, density=0.136, window=9,
                             window_mode=WINDOW_PRESERVE, seed=5),
    # the same 1536x2688 frames with the window at token level: 72 x 72 tokens = 1152 x 1152 px
    "uhr_truncate_tok": Workload("uhr_truncate_tok", B=1, H=12, D=128, Y=96, X=168, q_frames=2,
                                 kv_past=(4,), cap_frames=6, density=0.136, window=72,
                                 window_mode=WINDOW_TRUNCATE_TOKENS, seed=5),
    "uhr_preserve_tok": Workload("uhr_preserve_tok", B=1, H=12, D=128, Y=96, X=168, q_frames=2,
                                 kv_past=(4,), cap_frames=6, density=0.136, window=72,
                                 window_mode=WINDOW_PRESERVE_TOKENS, seed=5),
}


def workload(name: str) -> Workload:
    return WORKLOADS[name]


def small_variant(w: Workload, H: int = 2, Y: int = 24, X: int = 40, **kw) -> Workload:
    """Same recipe on fewer heads and a smaller token grid (for fast parity runs)."""
    return replace(w, name=w.name + "_small", H=H, Y=Y, X=X, **kw)


def _rope3d_(x: torch.Tensor, t0: int) -> None:
    """Rotate channel pairs in place by (t, y, x) positions, 44/42/42 channels.

    Input preparation only (the model's positional encoding, which the pages
    give as the reason for the locality window); the method never sees it.
    ``x`` is fp32 ``[H][F][Y][X][D]`` with D == 128; frame f has position t0+f.
    """
    H, F, Y, X, D = x.shape
    splits = (44, 42, 42)
    assert D == sum(splits)
    pos = (
        (torch.arange(F, dtype=torch.float64) + t0).view(F, 1, 1).expand(F, Y, X),
        torch.arange(Y, dtype=torch.float64).view(1, Y, 1).expand(F, Y, X),
        torch.arange(X, dtype=torch.float64).view(1, 1, X).expand(F, Y, X),
    )
    c0 = 0
    for n, p in zip(splits, pos):
        half = n // 2
        freq = 10000.0 ** (-2.0 * torch.arange(half, dtype=torch.float64) / n)
        ang = (p.unsqueeze(-1) * freq).to(torch.float32)  # [F][Y][X][half]
        cos, sin = torch.cos(ang), torch.sin(ang)
        a = x[..., c0:c0 + n:2].clone()
        b = x[..., c0 + 1:c0 + n:2].clone()
        x[..., c0:c0 + n:2] = a * cos - b * sin
        x[..., c0 + 1:c0 + n:2] = a * sin + b * cos
        c0 += n


def _field(g: torch.Generator, Y: int, X: int, D: int) -> torch.Tensor:
    """Smooth spatial field f_c(y,x) = cos(2*pi*(u_c*y/Y + v_c*x/X) + phi_c)."""
    u = torch.randint(0, 3, (D,), generator=g).to(torch.float32)
    v = torch.randint(0, 3, (D,), generator=g).to(torch.float32)
    phi = torch.rand(D, generator=g) * (2 * math.pi)
    yy = torch.arange(Y, dtype=torch.float32).view(Y, 1, 1)
    xx = torch.arange(X, dtype=torch.float32).view(1, X, 1)
    return torch.cos(2 * math.pi * (u * yy / Y + v * xx / X) + phi)  # [Y][X][D]


def make_inputs(w: Workload):
    """Draw Q, K, V for workload ``w``.

    Returns a dict with
      ``q``:  bf16 ``[B][H][q_frames][Y][X][D]`` (the current chunk of every stream)
      ``k``, ``v``: lists of bf16 ``[H][F_b][Y][X][D]``, the whole timeline of
             stream b (past frames then the chunk), F_b = kv_past[b] + q_frames.
    """
    g = torch.Generator(device="cpu").manual_seed(w.seed)
    field = _field(g, w.Y, w.X, w.D) if w.structure == "field" else None
    qs, ks, vs = [], [], []
    for b in range(w.B):
        F = w.kv_past[b] + w.q_frames
        q = torch.randn((w.H, w.q_frames, w.Y, w.X, w.D), generator=g)
        k = torch.randn((w.H, F, w.Y, w.X, w.D), generator=g)
        v = torch.randn((w.H, F, w.Y, w.X, w.D), generator=g)
        if w.structure == "rope":
            _rope3d_(q, t0=F - w.q_frames)
            _rope3d_(k, t0=0)
        elif w.structure == "field":
            q += field
            k += field
        qs.append(q.to(torch.bfloat16))
        ks.append(k.to(torch.bfloat16))
        vs.append(v.to(torch.bfloat16))
    return {"q": torch.stack(qs), "k": ks, "v": vs, "workload": w}


@dataclass(frozen=True)
class SegmentWorkload:
    """A batch of segments (video clips, or images as one-frame videos) for
    dense attention confined to each segment; ``seg_frames[b]`` latent frames
    in segment b, queries padded to the longest segment (padding frames are
    the oldest positions and hold zeros)."""

    name: str
    H: int
    D: int
    Y: int
    X: int
    seg_frames: Tuple[int, ...]
    seed: int = 0

    @property
    def B(self) -> int:
        return len(self.seg_frames)

    @property
    def q_frames(self) -> int:
        return max(self.seg_frames)

    @property
    def cap_frames(self) -> int:
        return self.q_frames + (self.q_frames & 1)


SEGMENT_WORKLOADS = {
    # two 21-frame video clips (6 latent frames), one 13-frame clip (4) and one image
    "joint": SegmentWorkload("joint", H=12, D=128, Y=48, X=88, seg_frames=(6, 6, 4, 1), seed=6),
}


def make_segment_inputs(w: SegmentWorkload):
    """Draw Q, K, V of every segment (N(0,1), rounded to bf16). Returns
    ``q`` bf16 ``[B][H][Tq][Y][X][D]`` (segment b in its newest seg_frames[b]
    frames, zeros before) and per-segment lists ``k``, ``v`` of
    ``[H][seg_frames[b]][Y][X][D]``."""
    g = torch.Generator(device="cpu").manual_seed(w.seed)
    Tq = w.q_frames
    q = torch.zeros((w.B, w.H, Tq, w.Y, w.X, w.D), dtype=torch.bfloat16)
    ks, vs = [], []
    for b, F in enumerate(w.seg_frames):
        q[b, :, Tq - F:] = torch.randn((w.H, F, w.Y, w.X, w.D), generator=g).to(torch.bfloat16)
        ks.append(torch.randn((w.H, F, w.Y, w.X, w.D), generator=g).to(torch.bfloat16))
        vs.append(torch.randn((w.H, F, w.Y, w.X, w.D), generator=g).to(torch.bfloat16))
    return {"q": q, "k": ks, "v": vs, "workload": w}


def stacked(frames: List[torch.Tensor]) -> torch.Tensor:
    """Stack per-stream timelines of equal length into ``[B][H][F][Y][X][D]``."""
    return torch.stack(frames)
