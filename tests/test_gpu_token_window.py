"""GPU parity of the token-level locality window: selections with token window
modes (candidates = key blocks that some token of the query block sees) match
the oracle bit for bit, and lcsa_sparse_attn_fwd_window (each query token sees
only the key tokens inside its window) matches the oracle's masked attention,
including query tokens that see no key at all (O = 0, LSE = -inf)."""
import numpy as np
import pytest
import torch

import lcsa_inputs as li
from oracle import lcsa_oracle as orc

from lcsa_harness import check_output, check_selection, oracle_head, params_of, run_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lc():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import block_sparse_causal_lcsa_b200 as m
    return m


def _check_o(go, ro, gl, rl, where):
    empty = ~np.isfinite(rl)
    assert np.array_equal(~np.isfinite(gl), empty), where + ": rows without a visible key differ"
    if empty.any():
        assert np.all(go[empty] == 0.0), where
    keep = ~empty
    check_output(go[keep], ro[keep], gl[keep], rl[keep], where)


SMALL = [
    li.small_variant(li.workload("uhr_truncate_tok"), H=2, Y=48, X=56, window=20),
    li.small_variant(li.workload("uhr_preserve_tok"), H=2, Y=48, X=56, window=20),
    li.small_variant(li.workload("uhr_truncate_tok"), H=1, Y=40, X=48, window=35),
    li.small_variant(li.workload("uhr_preserve_tok"), H=1, Y=40, X=48, window=72),   # wider than the frame
]


@pytest.mark.parametrize("w", SMALL, ids=["%s_w%d" % (w.name, w.window) for w in SMALL])
def test_token_window_every_row(lc, w):
    x = li.make_inputs(w)
    g = run_gpu(lc, w, x)
    assert g["err"] == 0
    for h in range(w.H):
        ref = oracle_head(w, x, 0, h)
        where = "%s h%d" % (w.name, h)
        check_selection(g["blk_idx"][0, h], g["blk_cnt"][0, h], ref["sel"], where)
        _check_o(g["O"][0, h], ref["O"], g["LSE"][0, h], ref["LSE"], where)


def test_rows_without_visible_keys(lc):
    """A 2-token window and one kept block per query block: most query tokens
    see none of its tokens."""
    w = li.Workload("tw_empty", B=1, H=1, D=128, Y=16, X=24, q_frames=2, kv_past=(2,), cap_frames=4,
                    top_k=1, window=2, window_mode=li.WINDOW_TRUNCATE_TOKENS, seed=51)
    x = li.make_inputs(w)
    g = run_gpu(lc, w, x)
    assert g["err"] == 0
    ref = oracle_head(w, x, 0, 0)
    check_selection(g["blk_idx"][0, 0], g["blk_cnt"][0, 0], ref["sel"], "empty rows")
    assert (~np.isfinite(ref["LSE"])).any()
    _check_o(g["O"][0, 0], ref["O"], g["LSE"][0, 0], ref["LSE"], "empty rows")


@pytest.mark.parametrize("name", ["uhr_truncate_tok", "uhr_preserve_tok"])
def test_full_size_token_window_selection_all_rows_output_sampled(lc, name):
    w = li.workload(name)
    x = li.make_inputs(w)
    g = run_gpu(lc, w, x)
    assert g["err"] == 0
    rng = np.random.default_rng(13)
    nQB = g["blk_cnt"].shape[2]
    rows = sorted(set(rng.choice(nQB, size=5, replace=False).tolist() + [0, 20, nQB - 1]))
    for h in (0, w.H - 1):
        ref = oracle_head(w, x, 0, h, rows=rows)
        where = "%s h%d" % (name, h)
        check_selection(g["blk_idx"][0, h], g["blk_cnt"][0, h], ref["sel"], where)
        O, L = g["O"][0, h], g["LSE"][0, h]
        mask = np.isfinite(ref["O"][..., 0]) | np.isinf(ref["LSE"])
        _check_o(O[mask], ref["O"][mask], L[mask], ref["LSE"][mask], where)
