"""Pins of the CPU reference attention (forward and backward).

Independent checks: torch's fused scaled_dot_product_attention in fp64 on the
CPU (a different library routine), torch autograd through it (automatic
differentiation, not the hand-derived formulas), central finite differences,
and the identities every softmax attention satisfies.
"""

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import attention as A
from oracle import mask as M


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def _sdpa(q, k, v, allowed=None):
    t = [torch.from_numpy(x)[None, None] for x in (q, k, v)]
    am = None if allowed is None else torch.from_numpy(allowed)[None, None]
    return F.scaled_dot_product_attention(*t, attn_mask=am)[0, 0].numpy()


@pytest.mark.parametrize("n,d", [(7, 4), (64, 16), (96, 64)])
def test_all_ones_mask_is_dense_attention(n, d):
    q, k, v = _rand((n, d), 1), _rand((n, d), 2), _rand((n, d), 3)
    o, lse = A.forward(q, k, v, np.ones((n, n), bool), 1 / np.sqrt(d))
    np.testing.assert_allclose(o, _sdpa(q, k, v), rtol=1e-12, atol=1e-12)
    S = q @ k.T / np.sqrt(d)
    np.testing.assert_allclose(lse, np.log(np.exp(S).sum(1)), rtol=1e-12)


@pytest.mark.parametrize("f,s,sink", [(8, 16, True), (8, 16, False), (64, 4, True), (5, 9, True)])
def test_radial_forward_matches_masked_sdpa(f, s, sink):
    d = 16
    n = f * s
    q, k, v = _rand((n, d), 4), _rand((n, d), 5), _rand((n, d), 6)
    m = M.token_mask(f, s, sink)
    o, lse = A.forward(q, k, v, m, 1 / np.sqrt(d))
    np.testing.assert_allclose(o, _sdpa(q, k, v, m), rtol=1e-11, atol=1e-12)
    # rows of P sum to one
    S = np.where(m, q @ k.T / np.sqrt(d), -np.inf)
    np.testing.assert_allclose(np.exp(S - lse[:, None]).sum(1), 1.0, rtol=1e-12)


def test_two_frames_radial_equals_dense():
    f, s, d = 2, 24, 8
    n = f * s
    q, k, v = _rand((n, d), 7), _rand((n, d), 8), _rand((n, d), 9)
    o, _ = A.radial_forward(q[None, None], k[None, None], v[None, None], f, s, sink=False)
    np.testing.assert_allclose(o[0, 0], _sdpa(q, k, v), rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("f,s,sink", [(8, 8, True), (6, 5, False), (16, 4, True)])
def test_backward_matches_autograd(f, s, sink):
    d = 8
    n = f * s
    q, k, v, do = (_rand((n, d), 10 + t) for t in range(4))
    m = M.token_mask(f, s, sink)
    scale = 1 / np.sqrt(d)
    o, lse = A.forward(q, k, v, m, scale)
    dq, dk, dv = A.backward(q, k, v, o, do, lse, m, scale)
    tq, tk, tv = (torch.from_numpy(x)[None, None].requires_grad_(True) for x in (q, k, v))
    out = F.scaled_dot_product_attention(tq, tk, tv, attn_mask=torch.from_numpy(m)[None, None])
    out.backward(torch.from_numpy(do)[None, None])
    np.testing.assert_allclose(dq, tq.grad[0, 0].numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dk, tk.grad[0, 0].numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dv, tv.grad[0, 0].numpy(), rtol=1e-10, atol=1e-12)


def test_backward_finite_differences():
    f, s, d = 4, 3, 3
    n = f * s
    q, k, v, do = (_rand((n, d), 20 + t) for t in range(4))
    m = M.token_mask(f, s, True)
    scale = 1 / np.sqrt(d)

    def loss(q_, k_, v_):
        o_, _ = A.forward(q_, k_, v_, m, scale)
        return float((o_ * do).sum())

    o, lse = A.forward(q, k, v, m, scale)
    grads = A.backward(q, k, v, o, do, lse, m, scale)
    eps = 1e-6
    for which, g in enumerate(grads):
        for (r, c) in [(0, 0), (n - 1, d - 1), (5, 1), (7, 2)]:
            args = [q.copy(), k.copy(), v.copy()]
            args[which][r, c] += eps
            up = loss(*args)
            args[which][r, c] -= 2 * eps
            dn = loss(*args)
            assert abs((up - dn) / (2 * eps) - g[r, c]) < 1e-7


def test_gradient_identities():
    """sum_b dS_ab = 0 for every row, hence column sums of dK vanish; and
    sum_b dV_b = sum_a dO_a (rows of P sum to one)."""
    f, s, d = 8, 8, 8
    n = f * s
    q, k, v, do = (_rand((n, d), 30 + t) for t in range(4))
    m = M.token_mask(f, s, True)
    scale = 1 / np.sqrt(d)
    o, lse = A.forward(q, k, v, m, scale)
    dq, dk, dv = A.backward(q, k, v, o, do, lse, m, scale)
    np.testing.assert_allclose(dk.sum(0), 0.0, atol=1e-11)
    np.testing.assert_allclose(dv.sum(0), do.sum(0), rtol=1e-11, atol=1e-11)


def test_row_sampled_paths_match_full():
    f, s, d = 8, 16, 16
    n = f * s
    q, k, v, do = (_rand((n, d), 40 + t) for t in range(4))
    m = M.token_mask(f, s, True)
    scale = 1 / np.sqrt(d)
    o, lse = A.forward(q, k, v, m, scale)
    dq, _, _ = A.backward(q, k, v, o, do, lse, m, scale)
    rows = A.sample_rows(n, 40, s, 16, seed=3)
    o_r, l_r = A.forward_rows(q, k, v, rows, f, s, True, chunk=7)
    np.testing.assert_allclose(o_r, o[rows], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(l_r, lse[rows], rtol=1e-12)
    np.testing.assert_allclose(A.dq_rows(q, k, v, do, rows, f, s, True, chunk=5), dq[rows],
                               rtol=1e-10, atol=1e-12)


def test_sample_rows_contains_edges():
    n, s, B = 1000, 100, 64
    rows = A.sample_rows(n, 200, s, B, seed=0)
    assert rows[0] == 0 and rows[-1] == n - 1
    assert 100 in rows and 99 in rows and (n // B) * B in rows
    assert np.all(np.diff(rows) > 0)
