"""Generate the coefficients of the polynomial exp2 used on the FMA pipe.

2^x = 2^j * 2^f with j = round(x) and f = x - j in [-1/2, 1/2] (Cody-Waite
style argument reduction); 2^f is approximated by a cubic p(f) whose
relative error is made (near) minimax by Lawson's iteratively reweighted
least squares.  The coefficients printed here are pasted into
attn_fwd.cuh; rerun to check them.
"""

import numpy as np


def fit(deg=3, lo=-0.5, hi=0.5, iters=400):
    g = np.linspace(lo, hi, 8001)
    t = 2.0 ** g
    A = np.stack([g ** k / t for k in range(deg + 1)], axis=1)
    b = np.ones_like(g)
    w = np.ones_like(g) / g.size
    for _ in range(iters):
        sw = np.sqrt(w)
        c, *_ = np.linalg.lstsq(A * sw[:, None], b * sw, rcond=None)
        e = A @ c - b
        w = w * np.abs(e)
        w /= w.sum()
    return c


def fp32_horner_error(c, lo=-0.5, hi=0.5):
    x = np.linspace(lo, hi, 1000001).astype(np.float32)
    c32 = c.astype(np.float32)
    acc = np.full_like(x, c32[-1])
    for k in range(len(c32) - 2, -1, -1):
        acc = acc * x + c32[k]
    ref = 2.0 ** x.astype(np.float64)
    return float(np.abs(acc.astype(np.float64) - ref).max() / 1.0), float((np.abs(acc - ref) / ref).max())


if __name__ == "__main__":
    c = fit()
    print("coefficients c0..c3 (fp32):", [float(np.float32(x)) for x in c])
    print("max abs / rel error of the fp32 Horner evaluation: %.3e / %.3e" % fp32_horner_error(c))
