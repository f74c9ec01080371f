"""Masked softmax attention, forward and backward -- plain CPU reference, fp64.

TEST INFRASTRUCTURE ONLY (see the package docstring): never imported by the
product path.

The method computes exactly (up to rounding order) the masked softmax
attention of [review] §3 Eq.2, ``O = softmax(Q K^T * scale + M) V`` with
``M`` = 0 on allowed pairs and -inf elsewhere; its block-sparse execution
([review] §4.2, 128x128 blocks) only skips tiles where ``M`` is -inf
everywhere.  So this module is that definition written out, with no blocking,
fusion or reordering.  The whole-head functions at the end evaluate each
chunk of rows against a superset of its allowed keys (mask.key_superset):
the keys they leave out are masked for every row of the chunk and would add
exp(-inf) = 0 to each sum, so the result is the same definition; the tests
pin them to the dense evaluation.  The pages fix neither the scale nor the saved
statistics; the readings taken: ``scale = 1/sqrt(d)`` (the Eq.1 convention),
``LSE`` = natural-log log-sum-exp of the masked, scaled logits per row.

Backward ([review] §4.3 uses the same attention under LoRA fine-tuning, so
its gradients are needed; the pages print no formulas): the plain
derivative of Eq.2 --
    P  = exp(S - LSE)                (S masked to -inf off the mask)
    dV = P^T dO
    dP = dO V^T
    Dr = rowsum(dO * O)
    dS = P * (dP - Dr)
    dQ = scale * dS K,   dK = scale * dS^T Q.

Every array is float64; callers pass bf16-rounded values where the device
consumes bf16 (the oracle then sees exactly the device's inputs).
"""

from __future__ import annotations

import numpy as np

from . import mask as _mask


def _as64(x):
    return np.asarray(x, dtype=np.float64)


def forward(q, k, v, allowed, scale):
    """[review] §3 Eq.2 for one (batch, head): q,k,v (n, d); allowed (n, n) bool.

    Returns (O (n, d), LSE (n,)).  A row with no allowed key gets O = 0,
    LSE = -inf (cannot happen under the radial mask: same-frame is dense).
    """
    q, k, v = _as64(q), _as64(k), _as64(v)
    S = (q @ k.T) * scale
    S = np.where(allowed, S, -np.inf)
    m = S.max(axis=1, keepdims=True)
    live = np.isfinite(m)
    m0 = np.where(live, m, 0.0)
    P = np.exp(S - m0)
    l = P.sum(axis=1, keepdims=True)
    with np.errstate(divide="ignore", invalid="ignore"):
        O = np.where(live, (P / np.where(live, l, 1.0)) @ v, 0.0)
        lse = np.where(live[:, 0], m0[:, 0] + np.log(np.where(live[:, 0], l[:, 0], 1.0)), -np.inf)
    return O, lse


def backward(q, k, v, o, do, lse, allowed, scale):
    """Gradients of Eq.2 for one (batch, head).  Returns (dQ, dK, dV)."""
    q, k, v, o, do, lse = (_as64(x) for x in (q, k, v, o, do, lse))
    S = (q @ k.T) * scale
    with np.errstate(invalid="ignore"):
        P = np.where(allowed, np.exp(S - lse[:, None]), 0.0)
    dV = P.T @ do
    dP = do @ v.T
    Dr = (do * o).sum(axis=1)
    dS = P * (dP - Dr[:, None])
    dQ = scale * (dS @ k)
    dK = scale * (dS.T @ q)
    return dQ, dK, dV


# ---------------------------------------------------------------------------
# Radial-mask wrappers over [B, H, N, D] arrays
# ---------------------------------------------------------------------------

def radial_forward(q, k, v, f, s, sink=True, scale=None, spec=None):
    """Eq.2 under the radial mask for every (batch, head) of [B, H, N, D] inputs."""
    q, k, v = _as64(q), _as64(k), _as64(v)
    Bn, H, N, D = q.shape
    assert N == f * s
    scale = 1.0 / np.sqrt(D) if scale is None else scale
    M = _mask.token_mask(f, s, sink, spec)
    O = np.empty_like(q)
    L = np.empty((Bn, H, N))
    for b in range(Bn):
        for h in range(H):
            O[b, h], L[b, h] = forward(q[b, h], k[b, h], v[b, h], M, scale)
    return O, L


def radial_backward(q, k, v, o, do, lse, f, s, sink=True, scale=None, spec=None):
    """Gradients under the radial mask for every (batch, head)."""
    q = _as64(q)
    Bn, H, N, D = q.shape
    scale = 1.0 / np.sqrt(D) if scale is None else scale
    M = _mask.token_mask(f, s, sink, spec)
    out = [np.empty_like(q) for _ in range(3)]
    for b in range(Bn):
        for h in range(H):
            g = backward(q[b, h], k[b, h], v[b, h], o[b, h], do[b, h], lse[b, h], M, scale)
            for t in range(3):
                out[t][b, h] = g[t]
    return tuple(out)


# ---------------------------------------------------------------------------
# Row-sampled evaluation (large shapes: each output row computed on its own)
# ---------------------------------------------------------------------------

def forward_rows(q, k, v, rows, f, s, sink=True, scale=None, chunk=256):
    """O and LSE of the given query rows of one (batch, head): q,k,v (n, d).

    Row r only needs its own logits against all keys, so it is Eq.2 applied to
    those rows alone.  Returns (O_rows (R, d), LSE_rows (R,)).
    """
    q, k, v = _as64(q), _as64(k), _as64(v)
    rows = np.asarray(rows, dtype=np.int64)
    scale = 1.0 / np.sqrt(q.shape[1]) if scale is None else scale
    O = np.empty((rows.size, q.shape[1]))
    L = np.empty(rows.size)
    for c0 in range(0, rows.size, chunk):
        r = rows[c0:c0 + chunk]
        M = _mask.row_mask(r, f, s, sink)
        S = (q[r] @ k.T) * scale
        S = np.where(M, S, -np.inf)
        m = S.max(axis=1, keepdims=True)
        P = np.exp(S - m)
        l = P.sum(axis=1, keepdims=True)
        O[c0:c0 + r.size] = (P / l) @ v
        L[c0:c0 + r.size] = m[:, 0] + np.log(l[:, 0])
    return O, L


def dq_rows(q, k, v, do, rows, f, s, sink=True, scale=None, chunk=256):
    """dQ of the given query rows of one (batch, head).

    dQ_r depends only on row r's own logits, its O_r, LSE_r and dO_r, all of
    which are recomputed here in fp64 from the inputs.
    """
    q, k, v, do = _as64(q), _as64(k), _as64(v), _as64(do)
    rows = np.asarray(rows, dtype=np.int64)
    scale = 1.0 / np.sqrt(q.shape[1]) if scale is None else scale
    out = np.empty((rows.size, q.shape[1]))
    for c0 in range(0, rows.size, chunk):
        r = rows[c0:c0 + chunk]
        M = _mask.row_mask(r, f, s, sink)
        S = np.where(M, (q[r] @ k.T) * scale, -np.inf)
        m = S.max(axis=1, keepdims=True)
        P = np.exp(S - m)
        P /= P.sum(axis=1, keepdims=True)
        o = P @ v
        dP = do[r] @ v.T
        Dr = (do[r] * o).sum(axis=1)
        dS = P * (dP - Dr[:, None])
        out[c0:c0 + r.size] = scale * (dS @ k)
    return out


def sample_rows(n, count, s, B, seed):
    """Seeded sample of query rows: first/last row, every frame-boundary row
    pair, the tail block, plus uniform random rows -- sorted, unique."""
    rng = np.random.default_rng(seed)
    fixed = [0, n - 1]
    for fb in range(s, n, s):
        fixed += [fb - 1, fb]
    tail0 = (n // B) * B
    fixed += list(range(tail0, n))
    fixed = np.unique(np.clip(np.asarray(fixed, dtype=np.int64), 0, n - 1))
    if fixed.size >= count:
        pick = rng.choice(fixed, size=count, replace=False)
        return np.sort(pick)
    extra = rng.choice(n, size=min(n, count * 2), replace=False)
    extra = np.setdiff1d(extra, fixed)[: count - fixed.size]
    return np.sort(np.concatenate([fixed, extra]))


def sample_runs(n, count, s, B, seed, run=64):
    """Seeded sample of about `count` query rows made of runs of `run`
    consecutive rows: the first and last rows, the tail block, a run across
    each of a random half-budget of frame boundaries, and random runs for the
    rest -- sorted, unique.  Runs let forward_runs / dq_runs evaluate many
    rows against one key superset."""
    rng = np.random.default_rng(seed)
    n_runs = max(1, count // run)
    starts = [0, max(0, n - run)]
    tail0 = (n // B) * B
    if tail0 < n:
        starts.append(tail0)
    bounds = np.arange(s, n, s, dtype=np.int64)
    if bounds.size:
        take = min(bounds.size, max(0, n_runs // 2))
        pick = rng.choice(bounds, size=take, replace=False) if take else np.zeros(0, np.int64)
        starts += [int(b) - run // 2 for b in pick]
    while len(starts) < n_runs:
        starts.append(int(rng.integers(0, max(1, n - run + 1))))
    rows = np.concatenate([np.arange(max(0, a), min(n, a + run), dtype=np.int64) for a in starts])
    return np.unique(rows)


def _runs_in_frames(rows, s, max_run):
    """Split sorted unique rows into [a0, a1) runs of consecutive rows inside
    one frame, at most max_run long."""
    rows = np.asarray(rows, dtype=np.int64)
    out = []
    i = 0
    while i < rows.size:
        a0 = int(rows[i])
        j = i + 1
        while (j < rows.size and rows[j] == rows[j - 1] + 1 and rows[j] // s == a0 // s
               and j - i < max_run):
            j += 1
        out.append((i, j, a0, int(rows[j - 1]) + 1))
        i = j
    return out


def forward_runs(q, k, v, rows, f, s, sink=True, scale=None, max_run=128, spec=None):
    """O and LSE of the given sorted query rows of one (batch, head): Eq.2
    evaluated for each run of consecutive rows of one frame against the run's
    key superset (mask.key_superset: every key it leaves out is masked for
    each row of the run, and adds exp(-inf) = 0).  Returns (O_rows, LSE_rows)."""
    k, v = _as64(k), _as64(v)
    rows = np.asarray(rows, dtype=np.int64)
    scale = 1.0 / np.sqrt(k.shape[1]) if scale is None else scale
    O = np.empty((rows.size, k.shape[1]))
    L = np.empty(rows.size)
    for i0, i1, a0, a1 in _runs_in_frames(rows, s, max_run):
        keys = _mask.key_superset(a0, a1, f, s, sink, spec)
        r = rows[i0:i1]
        S = (_as64(q[r]) @ k[keys].T) * scale
        S = np.where(_mask.pair_mask(r, keys, f, s, sink, spec), S, -np.inf)
        m = S.max(axis=1, keepdims=True)
        P = np.exp(S - m)
        l = P.sum(axis=1, keepdims=True)
        O[i0:i1] = (P @ v[keys]) / l
        L[i0:i1] = m[:, 0] + np.log(l[:, 0])
    return O, L


def dq_runs(q, k, v, do, rows, f, s, sink=True, scale=None, max_run=128, spec=None):
    """dQ of the given sorted query rows of one (batch, head), run by run as
    forward_runs (each row's O, LSE and rowsum(dO o O) recomputed in fp64)."""
    k, v = _as64(k), _as64(v)
    rows = np.asarray(rows, dtype=np.int64)
    scale = 1.0 / np.sqrt(k.shape[1]) if scale is None else scale
    out = np.empty((rows.size, k.shape[1]))
    for i0, i1, a0, a1 in _runs_in_frames(rows, s, max_run):
        keys = _mask.key_superset(a0, a1, f, s, sink, spec)
        r = rows[i0:i1]
        kk, vv = k[keys], v[keys]
        S = np.where(_mask.pair_mask(r, keys, f, s, sink, spec), (_as64(q[r]) @ kk.T) * scale, -np.inf)
        m = S.max(axis=1, keepdims=True)
        P = np.exp(S - m)
        P /= P.sum(axis=1, keepdims=True)
        dor = _as64(do[r])
        o = P @ vv
        dS = P * (dor @ vv.T - (dor * o).sum(axis=1)[:, None])
        out[i0:i1] = scale * (dS @ kk)
    return out


# ---------------------------------------------------------------------------
# Whole-head statistics and key-column gradients (dK, dV at large shapes)
# ---------------------------------------------------------------------------

def _chunks_in_frames(n, s, chunk):
    """Consecutive row ranges [a0, a1) of at most `chunk` rows, none crossing
    a frame boundary."""
    out = []
    for f0 in range(0, n, s):
        f1 = min(n, f0 + s)
        for a0 in range(f0, f1, chunk):
            out.append((a0, min(f1, a0 + chunk)))
    return out


def head_row_stats(q, k, v, do, f, s, sink=True, scale=None, chunk=128, threads=None, spec=None):
    """LSE and Dr = rowsum(dO * O) of EVERY query row of one (batch, head).

    Each chunk of consecutive rows of one frame is Eq.2 evaluated against
    the key superset of mask.key_superset(): the keys left out are masked
    for every row of the chunk, so they contribute exp(-inf) = 0 to every
    sum and leaving them out changes neither LSE nor O.  q, k, v, do: (n, d)
    arrays (any float dtype; the arithmetic is fp64).  Chunks run on a thread
    pool (NumPy releases the interpreter lock inside its kernels)."""
    import os
    from concurrent.futures import ThreadPoolExecutor

    n, dh = q.shape
    scale = 1.0 / np.sqrt(dh) if scale is None else scale
    q, k, v, do = (_as64(x) for x in (q, k, v, do))
    lse = np.empty(n)
    dr = np.empty(n)

    def work(rng):
        a0, a1 = rng
        keys = _mask.key_superset(a0, a1, f, s, sink, spec)
        rows = np.arange(a0, a1, dtype=np.int64)
        S = q[a0:a1] @ k[keys].T
        S *= scale
        np.copyto(S, -np.inf, where=~_mask.pair_mask(rows, keys, f, s, sink, spec))
        m = S.max(axis=1, keepdims=True)
        S -= m
        np.exp(S, out=S)                       # S now holds P = exp(S - m)
        l = S.sum(axis=1, keepdims=True)
        o = (S @ v[keys]) / l
        lse[a0:a1] = m[:, 0] + np.log(l[:, 0])
        dr[a0:a1] = (do[a0:a1] * o).sum(axis=1)

    ranges = _chunks_in_frames(n, s, chunk)
    threads = threads or max(1, len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else 1)
    try:
        from threadpoolctl import threadpool_limits
        limiter = threadpool_limits(1)
    except Exception:  # pragma: no cover - threadpoolctl is optional
        limiter = None
    try:
        with ThreadPoolExecutor(threads) as ex:
            list(ex.map(work, ranges))
    finally:
        if limiter is not None:
            limiter.restore_original_limits()
    return lse, dr


def dkdv_cols(q, k, v, do, lse, dr, cols, f, s, sink=True, scale=None, chunk=8192, threads=None, spec=None):
    """dK and dV of the given key columns of one (batch, head).

    Column b of the gradients is a sum over every query a:
        P[a, b] = exp(S[a, b] - LSE[a])  (0 where (a, b) is masked)
        dV[b]   = sum_a P[a, b] dO[a]
        dS[a, b] = P[a, b] (dO[a] . V[b] - Dr[a])
        dK[b]   = scale * sum_a dS[a, b] Q[a]
    with the row statistics LSE and Dr of every query (head_row_stats or the
    dense forward).  Queries are taken in chunks; the result is a plain sum
    over them (chunks on a thread pool, partial sums added in query order).
    Returns (dK_cols, dV_cols), each (len(cols), d)."""
    import os
    from concurrent.futures import ThreadPoolExecutor

    n, dh = q.shape
    scale = 1.0 / np.sqrt(dh) if scale is None else scale
    cols = np.asarray(cols, dtype=np.int64)
    kc, vc = _as64(k[cols]), _as64(v[cols])

    def part(a0):
        a1 = min(n, a0 + chunk)
        rows = np.arange(a0, a1, dtype=np.int64)
        qa, doa = _as64(q[a0:a1]), _as64(do[a0:a1])
        S = (qa @ kc.T) * scale
        with np.errstate(invalid="ignore", over="ignore"):
            P = np.where(_mask.pair_mask(rows, cols, f, s, sink, spec),
                         np.exp(S - _as64(lse[a0:a1])[:, None]), 0.0)
        dS = P * (doa @ vc.T - _as64(dr[a0:a1])[:, None])
        return dS.T @ qa, P.T @ doa

    threads = threads or max(1, len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else 1)
    try:
        from threadpoolctl import threadpool_limits
        limiter = threadpool_limits(1)
    except Exception:  # pragma: no cover - threadpoolctl is optional
        limiter = None
    try:
        with ThreadPoolExecutor(threads) as ex:
            parts = list(ex.map(part, range(0, n, chunk)))   # in query order
    finally:
        if limiter is not None:
            limiter.restore_original_limits()
    dK = np.zeros((cols.size, dh))
    dV = np.zeros((cols.size, dh))
    for pk, pv in parts:
        dK += pk
        dV += pv
    return scale * dK, dV
