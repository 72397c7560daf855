"""Seeded input generators: shapes, dtypes, determinism, workload recipes."""
import torch

import lcsa_inputs as li


def test_workload_shapes_and_recipes():
    w = li.workload("chunk")
    assert (w.H, w.D, w.Y, w.X, w.q_frames, w.kv_frames) == (12, 128, 48, 88, 2, (6,))
    assert (w.Hb, w.Wb) == (6, 11)
    u = li.workload("uhr_preserve")
    assert (u.Y, u.X, u.Hb, u.Wb, u.window) == (96, 168, 12, 21, 9)
    c = li.workload("clip")
    assert c.q_frames == 26 and c.kv_frames == (26,) and c.Y * c.X * 26 == 109824
    m = li.workload("multistream")
    assert m.B == 4 and set(m.kv_past) == {4, 5, 6} and m.cap_frames == 8


def test_inputs_are_seeded_bf16():
    w = li.small_variant(li.workload("multistream"), H=1, Y=16, X=16)
    a, b = li.make_inputs(w), li.make_inputs(w)
    assert a["q"].dtype == torch.bfloat16 and a["q"].shape == (4, 1, 2, 16, 16, 128)
    for b_, F in enumerate(w.kv_frames):
        assert a["k"][b_].shape == (1, F, 16, 16, 128)
        assert torch.equal(a["k"][b_], b["k"][b_]) and torch.equal(a["v"][b_], b["v"][b_])
    assert torch.equal(a["q"], b["q"])


def test_rope_and_field_structure_change_values_only():
    for name in ("chunk", "clip"):
        w = li.small_variant(li.workload(name), H=1, Y=16, X=16)
        x = li.make_inputs(w)
        assert torch.isfinite(x["q"].float()).all()
        # the structure is shared by Q and K (same positions / same field), V is plain N(0,1)
        assert abs(float(x["v"][0].float().std()) - 1.0) < 0.05
