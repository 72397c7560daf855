"""GPU parity of dense attention confined to segments (the stage-1
block-diagonal segment mask; images are one-frame segments): the block lists of
lcsa_segment_blocks fed to lcsa_sparse_attn_fwd / lcsa_sparse_attn_bwd against
the fp64 oracle's segment_attention (and its backward), on ragged segments with
padded queries. Block lists are checked exactly; outputs within the forward
and backward tolerances of the other parity tests."""
import numpy as np
import pytest
import torch

import lcsa_inputs as li
from oracle import lcsa_oracle as orc

from lcsa_harness import check_output

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lc():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import block_sparse_causal_lcsa_b200 as m
    return m


def _setup(lc, w):
    x = li.make_segment_inputs(w)
    cache = lc.KVCache(w.B, w.H, w.cap_frames, w.Y, w.X, w.D)
    for b in range(w.B):
        lc.kv_append(cache, x["k"][b].unsqueeze(0).cuda(), x["v"][b].unsqueeze(0).cuda(), stream_offset=b)
    q = x["q"].cuda()
    idx, cnt = lc.segment_blocks(w.q_frames, cache)
    return x, cache, q, idx, cnt


def _ring(cache, t, b, h):
    lo, hi = cache.state()[b]
    return torch.stack([t[b, h, f % cache.cap_frames] for f in range(lo, hi)]).double().cpu().numpy()


SEGS = [li.SegmentWorkload("segs", H=2, D=128, Y=16, X=24, seg_frames=(6, 4, 1, 3), seed=41),
        li.SegmentWorkload("segs64", H=1, D=64, Y=24, X=16, seg_frames=(5, 2), seed=43)]


@pytest.mark.parametrize("w", SEGS, ids=[w.name for w in SEGS])
def test_segment_lists_forward_and_backward(lc, w):
    x, cache, q, idx, cnt = _setup(lc, w)
    o, lse = lc.sparse_attn_fwd(q, cache, idx, cnt)
    g = torch.Generator().manual_seed(5)
    d_o = torch.randn(q.shape, generator=g).to(torch.bfloat16)   # host; the oracle reads this copy
    Tq = w.q_frames
    for b, F in enumerate(w.seg_frames):
        d_o[b, :, :Tq - F] = 0          # padding rows carry no gradient
    dq, dk, dv = lc.sparse_attn_bwd(q, cache, idx, cnt, o, lse, d_o.cuda())
    torch.cuda.synchronize()
    assert lc.last_device_error() == 0
    Hb, Wb = w.Y // 8, w.X // 8
    nQT = (Tq + 1) // 2
    for b, F in enumerate(w.seg_frames):
        nkb = ((F + 1) // 2) * Hb * Wb
        for h in range(w.H):
            # block lists: every key block of the segment for blocks holding a segment frame, none for padding
            for i in range(nQT * Hb * Wb):
                newer = Tq - 2 * nQT + 2 * (i // (Hb * Wb)) + 1
                want = nkb if newer >= Tq - F else 0
                assert int(cnt[b, h, i]) == want
                assert torch.equal(idx[b, h, i, :want].cpu(), torch.arange(want, dtype=torch.int32))
            qs = orc.widen(x["q"][b, h, Tq - F:])
            ks, vs = orc.widen(x["k"][b][h]), orc.widen(x["v"][b][h])
            ro, rl = orc.segment_attention(qs, ks, vs)
            check_output(o[b, h, Tq - F:].double().cpu().numpy(), ro, lse[b, h, Tq - F:].double().cpu().numpy(), rl,
                         "%s b%d h%d" % (w.name, b, h))
            rq, rk, rv = orc.segment_attention_backward(qs, ks, vs, orc.widen(d_o[b, h, Tq - F:]))
            for got, ref, name in ((dq[b, h, Tq - F:].double().cpu().numpy(), rq, "dq"),
                                   (_ring(cache, dk, b, h), rk, "dk"), (_ring(cache, dv, b, h), rv, "dv")):
                rel = np.linalg.norm(got - ref) / np.linalg.norm(ref)
                assert rel <= 2e-2, "%s b%d h%d %s rel-L2 %.3g" % (w.name, b, h, name, rel)


def test_full_size_joint_batch_sampled(lc):
    """The 768x1408 joint batch (two 6-frame clips, a 4-frame clip, an image):
    outputs of sampled query blocks of two heads against the oracle."""
    w = li.SEGMENT_WORKLOADS["joint"]
    x, cache, q, idx, cnt = _setup(lc, w)
    o, lse = lc.sparse_attn_fwd(q, cache, idx, cnt)
    torch.cuda.synchronize()
    assert lc.last_device_error() == 0
    Tq = w.q_frames
    for b, F in enumerate(w.seg_frames):
        for h in (0, w.H - 1):
            qs = orc.widen(x["q"][b, h, Tq - F:])
            # the first 8 token rows of the segment's newest frame (the oracle on all rows is slow)
            ro, rl = orc.segment_attention(qs[-1:, :8], orc.widen(x["k"][b][h]), orc.widen(x["v"][b][h]))
            check_output(o[b, h, Tq - 1:, :8].double().cpu().numpy(), ro,
                         lse[b, h, Tq - 1:, :8].double().cpu().numpy(), rl, "joint b%d h%d" % (b, h))
