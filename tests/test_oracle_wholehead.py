"""The oracle's whole-head evaluation (used by the large-shape dK / dV parity
checks) against its dense definition.

mask.key_superset must contain every allowed key of its rows (checked
against the brute-force token mask); head_row_stats must give the LSE and
rowsum(dO o O) of the dense forward; dkdv_cols must give the dense backward's
dK and dV columns.  The dense functions are themselves pinned to textbook
attention, autograd and finite differences (test_oracle_attention.py)."""

import numpy as np
import pytest

from oracle import attention as A
from oracle import mask as M


@pytest.mark.parametrize("f,s,sink,chunk", [
    (9, 30, True, 7), (9, 30, False, 30), (40, 3, True, 2), (64, 4, False, 3),
    (5, 200, True, 64), (1, 50, False, 16), (33, 12, True, 5)])
def test_key_superset_contains_every_allowed_key(f, s, sink, chunk):
    full = M.token_mask(f, s, sink)
    n = f * s
    for a0, a1 in A._chunks_in_frames(n, s, chunk):
        keys = M.key_superset(a0, a1, f, s, sink)
        assert np.all(np.diff(keys) > 0)
        allowed_keys = np.nonzero(full[a0:a1].any(axis=0))[0]
        assert np.isin(allowed_keys, keys).all(), (a0, a1)


def test_key_superset_is_much_smaller_than_n_for_far_frames():
    # the point of the superset: a chunk of one frame needs only a window of
    # the frames it reaches (f = 40, s = 256: far bands keep 1/8 .. 1/16 of a frame)
    f, s = 40, 256
    keys = M.key_superset(10 * s + 64, 10 * s + 96, f, s, True)
    assert keys.size < 0.6 * f * s


@pytest.mark.parametrize("f,s,sink,seed", [(9, 30, True, 1), (40, 3, True, 2), (64, 4, False, 3),
                                           (6, 50, False, 4)])
def test_head_row_stats_and_dkdv_cols_equal_dense(f, s, sink, seed):
    rng = np.random.default_rng(seed)
    n, d = f * s, 16
    q, k, v, do = (rng.standard_normal((n, d)) for _ in range(4))
    scale = 1.0 / np.sqrt(d)
    allowed = M.token_mask(f, s, sink)
    o, lse = A.forward(q, k, v, allowed, scale)
    dr = (do * o).sum(axis=1)
    lse2, dr2 = A.head_row_stats(q, k, v, do, f, s, sink, chunk=7, threads=3)
    np.testing.assert_allclose(lse2, lse, rtol=0, atol=1e-12)
    np.testing.assert_allclose(dr2, dr, rtol=0, atol=1e-12)
    _, dk, dv = A.backward(q, k, v, o, do, lse, allowed, scale)
    cols = np.sort(rng.choice(n, size=min(n, 37), replace=False))
    dk2, dv2 = A.dkdv_cols(q, k, v, do, lse2, dr2, cols, f, s, sink, chunk=19)
    np.testing.assert_allclose(dk2, dk[cols], rtol=0, atol=1e-12)
    np.testing.assert_allclose(dv2, dv[cols], rtol=0, atol=1e-12)


def test_dkdv_cols_planted_wrong_statistics_fail():
    """A plausible slip -- Dr taken from a different row -- changes dK."""
    f, s, d = 9, 30, 16
    rng = np.random.default_rng(7)
    n = f * s
    q, k, v, do = (rng.standard_normal((n, d)) for _ in range(4))
    lse, dr = A.head_row_stats(q, k, v, do, f, s, True)
    cols = np.arange(0, n, 11)
    dk, _ = A.dkdv_cols(q, k, v, do, lse, dr, cols, f, s, True)
    dk_bad, _ = A.dkdv_cols(q, k, v, do, lse, np.roll(dr, 1), cols, f, s, True)
    assert np.abs(dk - dk_bad).max() > 1e-3


@pytest.mark.parametrize("f,s,sink,seed", [(9, 30, True, 1), (40, 3, True, 2), (64, 4, False, 3),
                                           (6, 50, False, 4), (12, 17, True, 5)])
def test_forward_runs_and_dq_runs_equal_dense(f, s, sink, seed):
    rng = np.random.default_rng(seed)
    n, d = f * s, 16
    q, k, v, do = (rng.standard_normal((n, d)) for _ in range(4))
    scale = 1.0 / np.sqrt(d)
    allowed = M.token_mask(f, s, sink)
    o, lse = A.forward(q, k, v, allowed, scale)
    dq, _, _ = A.backward(q, k, v, o, do, lse, allowed, scale)
    rows = A.sample_runs(n, 60, s, 16, seed=seed, run=8)
    o2, l2 = A.forward_runs(q, k, v, rows, f, s, sink, max_run=5)
    np.testing.assert_allclose(o2, o[rows], rtol=0, atol=1e-12)
    np.testing.assert_allclose(l2, lse[rows], rtol=0, atol=1e-12)
    np.testing.assert_allclose(A.dq_runs(q, k, v, do, rows, f, s, sink, max_run=5), dq[rows], rtol=0, atol=1e-12)


def test_sample_runs_cover_the_edges():
    f, s, B = 20, 50, 16
    n = f * s
    rows = A.sample_runs(n, 400, s, B, seed=0, run=16)
    assert np.all(np.diff(rows) > 0) and rows[0] == 0 and rows[-1] == n - 1
    tail0 = (n // B) * B
    assert np.isin(np.arange(tail0, n), rows).all()
    # runs that straddle frame boundaries
    straddle = [b for b in range(s, n, s) if b - 1 in rows and b in rows]
    assert len(straddle) >= 5
    assert 300 <= rows.size <= 520
