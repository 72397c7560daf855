"""Fit the polynomial the attention kernel uses for part of its exp2 work.

The softmax of the sparse-attention kernel evaluates 2^x for x <= 8. Part of
those evaluations run on the FMA pipe instead of the special-function unit:
Cody-Waite style range reduction x = n + f with n = round(x), f in [-1/2, 1/2],
then 2^x = 2^n * p(f), the 2^n applied by adding n to the float's exponent
field. p is the degree-3 polynomial that minimises the maximum RELATIVE error
|p(f) / 2^f - 1| on [-1/2, 1/2], found here with the Remez exchange algorithm
(equioscillation on 5 points) in float64, then rounded to float32.

    python block_sparse_causal_lcsa_b200/csrc/fit_exp2_poly.py

prints the coefficients c0..c3 (p(f) = c0 + c1 f + c2 f^2 + c3 f^3) and the
float32 evaluation error; the constants in attn_fwd.cuh come from this output.
P is rounded to bf16 afterwards (relative error up to 2^-9), so a relative
error near 1e-4 is far below what the kernel keeps.
"""
import numpy as np

DEG = 3
LO, HI = -0.5, 0.5


def remez(deg=DEG, iters=30):
    # initial reference: Chebyshev extrema
    k = np.arange(deg + 2)
    x = 0.5 * (LO + HI) + 0.5 * (HI - LO) * np.cos(np.pi * k[::-1] / (deg + 1))
    for _ in range(iters):
        # solve p(x_i) - 2^x_i = (-1)^i E 2^x_i  (relative equioscillation)
        A = np.zeros((deg + 2, deg + 2))
        for i, xi in enumerate(x):
            A[i, :deg + 1] = xi ** np.arange(deg + 1)
            A[i, deg + 1] = -((-1) ** i) * 2.0 ** xi
        sol = np.linalg.solve(A, 2.0 ** x)
        c = sol[:deg + 1]
        # new reference: extrema of the relative error on a fine grid
        g = np.linspace(LO, HI, 200001)
        err = np.polyval(c[::-1], g) / 2.0 ** g - 1.0
        # split the grid at sign changes and take the extremum of each run
        s = np.sign(err)
        cuts = np.nonzero(np.diff(s))[0] + 1
        runs = np.split(np.arange(len(g)), cuts)
        ext = [r[np.argmax(np.abs(err[r]))] for r in runs if len(r)]
        if len(ext) >= deg + 2:
            # keep deg+2 alternating extrema with the largest magnitudes
            while len(ext) > deg + 2:
                mags = np.abs(err[ext])
                drop = 0 if mags[0] < mags[-1] else len(ext) - 1
                ext.pop(drop)
            x = g[ext]
    return c, np.max(np.abs(err))


def eval_f32(c, x):
    """The kernel's float32 evaluation: reduction, Horner, exponent add."""
    c = c.astype(np.float32)
    x = np.maximum(x.astype(np.float32), np.float32(-126.0))
    magic = np.float32(12582912.0)  # 1.5 * 2^23
    t = (x + magic).astype(np.float32)
    n = (t - magic).astype(np.float32)
    f = (x - n).astype(np.float32)
    p = np.float32(c[3])
    for ci in (c[2], c[1], c[0]):
        p = (p * f + ci).astype(np.float32)  # the kernel fuses these multiply-adds
    bits = p.view(np.int32) + (t.view(np.int32) << 23)
    return bits.view(np.float32)


if __name__ == "__main__":
    c, e = remez()
    print("minimax relative error (float64 coefficients): %.3e" % e)
    c32 = c.astype(np.float32)
    for i, v in enumerate(c32):
        print("c%d = %.9ef  (0x%08x)" % (i, v, np.array(v).view(np.uint32)))
    x = np.linspace(-100.0, 8.0, 2000001)
    y = eval_f32(c32.astype(np.float64), x)
    rel = np.abs(y.astype(np.float64) / 2.0 ** x - 1.0)
    print("float32 evaluation, x in [-100, 8]: max relative error %.3e" % rel.max())
