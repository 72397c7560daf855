"""The exp2 polynomial of the attention kernel, checked on the CPU: the Remez
fit reproduces the coefficients compiled into the kernel and its float32
evaluation meets the stated bound."""
import importlib.util
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "block_sparse_causal_lcsa_b200", "csrc")


def _fit_module():
    spec = importlib.util.spec_from_file_location("fit_exp2_poly", os.path.join(CSRC, "fit_exp2_poly.py"))
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    return m


def test_fit_matches_kernel_constants_and_bound():
    m = _fit_module()
    c, err = m.remez()
    assert err < 8e-5
    src = open(os.path.join(CSRC, "lcsa_device.cuh")).read()
    body = src[src.index("exp2_poly_f2"):]
    body = body[:body.index("return f2_pack(r0, r1)")]
    # the last four packed constants of the function are the Horner coefficients c3, c2, c1, c0
    consts = [float(v) for v in re.findall(r"f2_pack\(([0-9.e+-]+)f, \1f\)", body)][-4:]
    # Horner order in the kernel: c3, c2, c1, c0
    assert np.allclose(consts, np.float32(c[::-1]), rtol=0, atol=1e-9)
    x = np.linspace(-100.0, 8.0, 400001)
    y = m.eval_f32(np.float32(c), x)
    assert np.max(np.abs(y / 2.0 ** x - 1.0)) < 1e-4
    # the clamp keeps the exponent field non-negative: tiny, finite, non-negative
    z = m.eval_f32(np.float32(c), np.array([-np.inf, -1e30, -300.0, -127.0, -126.4]))
    assert np.isfinite(z).all() and (z >= 0).all() and (z < 1e-37).all()
