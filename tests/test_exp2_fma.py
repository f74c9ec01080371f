"""The softmax's FMA-pipe exponential (exp2_fma_x2 in sm100_primitives.cuh):
its cubic's coefficients are re-derived here from their definition -- a
least-squares fit of 2^f on [-1/2, 1/2] in relative error, reweighted towards
equal ripple (Lawson's iteration) -- and the constants in the header must
match them, with a maximum relative error below 1e-4 (bf16 P needs 2^-9)."""

import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _fit():
    f = np.linspace(-0.5, 0.5, 20001)
    y = np.exp2(f)
    V = np.vstack([f ** k for k in range(4)]).T
    w = np.ones_like(f)
    for _ in range(200):
        W = w / y
        c, *_ = np.linalg.lstsq(V * W[:, None], y * W, rcond=None)
        err = np.abs(V @ c - y) / y
        w = w * (err / err.max()) + 1e-30
        w /= w.sum()
    return c.astype(np.float32), f, y, V


def _header_coeffs():
    src = open(os.path.join(ROOT, "block_sparse_attention_csr_b200", "csrc", "sm100_primitives.cuh")).read()
    body = src[src.index("exp2_fma_x2(uint64_t x)"):]
    body = body[:body.index("\n}\n")]
    nums = [float(x) for x in re.findall(r"f2_pack\(([0-9.]+)f, \1f\)", body)]
    c3, c2, c1, c0 = nums[1:5]   # nums[0] is the 1.5 * 2^23 shift
    return np.array([c0, c1, c2, c3], dtype=np.float32)


def test_header_coefficients_are_the_fit():
    c, f, y, V = _fit()
    h = _header_coeffs()
    np.testing.assert_allclose(h, c, rtol=2e-6, atol=0)
    err = np.abs(V @ h.astype(np.float64) - y) / y
    assert err.max() < 1e-4
    # Horner in fp32, as the device evaluates it
    ff = f.astype(np.float32)
    p = ((h[3] * ff + h[2]) * ff + h[1]) * ff + h[0]
    assert (np.abs(p.astype(np.float64) - y) / y).max() < 1.2e-4
