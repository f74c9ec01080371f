"""Radial Attention static spatiotemporal mask -- plain CPU reference.

TEST INFRASTRUCTURE ONLY (see the package docstring): never imported by the
product path.

What the pages fix, and the readings taken where they are silent
----------------------------------------------------------------
Token layout ([review] §4, toy example): ``n = f * s`` tokens, frame-major;
token ``a = i*s + k`` is position ``k`` (row-major over the spatial grid) of
frame ``i``.  The 4D mask ``M~[i, j, k, l]`` is flattened to the 2D mask by
``M[i*s + k, j*s + l] = M~[i, j, k, l]`` ([review] §4.2, the flattening step;
the printed formula was lost, this is its plain reading).

Temporal bands ([review] §4.2, Fig.5a): the band of a frame pair is
``r(d) = floor(log2(max(d, 1)))`` with ``d = |i - j|``; density halves from one
band to the next, so frame distances 0 and 1 form the dense central band
(the [rebuttal] "width of central band" ablation: default 1 means
``|i - j| <= 1`` is dense).

Spatial diagonal ([review] §4.2, Fig.5b; toy example case C): inside the
frame-pair block the kept width is ``w(d) = floor(s / 2**r(d))``; the toy
example (s = 9, d = 2, w = 4, query position 4 keeps "roughly l = 1..7")
is reproduced exactly by keeping ``|k - l| <= h(d)`` with
``h(d) = w(d) - 1``.

Width below one ([review] Fig.5 caption and Eq.4 case (ii); [rebuttal]
"reduce the diagonal frequency when the width is below 1"): when
``w(d) = 0`` (``h(d) < 0``) only the main diagonal ``k == l`` is kept, and only
in every ``c(d)``-th frame pair, ``c(d) = ceil(2**r(d) / s)``, so the amortised
density keeps halving per band.  The exact subsampling rule is not printed;
``d mod c(d) == 0`` is the plainest reading.  What the pages do state -- the
amortised density keeps halving per band and only the main diagonal is kept
-- is pinned by brute-force band counts (tests/test_oracle_mask.py); which
frame pairs of a band carry the kept diagonal (the phase of ``d mod c``) is
the one choice the pages leave open.  The branch never triggers at the
benchmark shapes.

Attention sink ([review] §4.2 and App. A.1 Eq.8): every query also attends
to every token of frame 0 (key frame ``j == 0``).  Query rows of frame 0 are
not made dense by it.  ``sink`` is a flag (the [rebuttal] ablation turns it
off).

Blocks ([review] §4.2, "128x128 blocks"): a (query-block, key-block) tile is
ACTIVE iff it holds at least one allowed pair of in-range tokens; FULL iff
both blocks lie inside ``[0, n)`` and all ``B*B`` pairs are allowed; else
PARTIAL.  Tokens at or beyond ``n`` are neither rows nor allowed keys.

Two independent routes to the block tiles are provided: brute force over
the token mask (tiny shapes only) and a per-frame-segment interval test that
scales to the benchmark shapes; the tests pin the second to the first.
"""

from __future__ import annotations

from dataclasses import dataclass

import numpy as np

TILE_FULL = 1
TILE_PARTIAL = 2


# ---------------------------------------------------------------------------
# Per-frame-distance quantities ([review] §4.2, Fig.5 a/b, Eq.4)
# ---------------------------------------------------------------------------

def band_index(d):
    """r(d) = floor(log2(max(d, 1))) for integer frame distances d >= 0."""
    d = np.maximum(np.asarray(d, dtype=np.int64), 1)
    # frexp: d = m * 2**e with 0.5 <= m < 1, exact for integers < 2**53.
    return (np.frexp(d.astype(np.float64))[1] - 1).astype(np.int64)


def diag_width(d, s):
    """w(d) = floor(s / 2**r(d)): the kept diagonal width of frame pair distance d."""
    r = band_index(d)
    return np.asarray(s, dtype=np.int64) // (np.int64(1) << r)


def half_width(d, s):
    """h(d) = w(d) - 1: keep |k - l| <= h(d) inside the frame-pair block."""
    return diag_width(d, s) - 1


def sample_period(d, s):
    """c(d) = ceil(2**r(d) / s): frame-pair period of the sampled diagonal."""
    p = np.int64(1) << band_index(d)
    return (p + np.int64(s) - 1) // np.int64(s)


def distance_table(f, s):
    """(h, c) for every frame distance d in [0, f)."""
    d = np.arange(f, dtype=np.int64)
    return half_width(d, s), sample_period(d, s)


# ---------------------------------------------------------------------------
# Ablation variants ([rebuttal]: width of the central band, width scale
# between consecutive bands; [review] App. C.3: harmonic-series decay)
# ---------------------------------------------------------------------------

@dataclass(frozen=True)
class MaskSpec:
    """Mask family.  central_band: frame distances <= it are dense ([rebuttal]
    "a central band width of d means attention between frames i and j where
    |i - j| <= d", default 1).  Width scale sigma = scale_num / scale_den > 1
    between consecutive temporal bands ([rebuttal], default 2).  decay:
    "radial" (exponential bands, the method) or "harmonic" ([review] App. C.3:
    width inversely proportional to the distance from the diagonal).

    Readings (the pages print no formula for the variants):
      radial:   dist <= cb -> dense; else band r >= 1 with
                (cb+1) sigma^(r-1) <= dist < (cb+1) sigma^r, width
                w = floor(s / sigma^r).  cb = 1, sigma = 2 gives exactly
                r = floor(log2 dist), w = floor(s / 2^r) (the default rule).
      harmonic: dist <= cb -> dense; else e = dist - cb + 1, w = floor(s / e).
    In both, h = w - 1, and when w = 0 the diagonal k == l is kept in every
    c-th frame pair, c = ceil(s_eff / s) with s_eff = sigma^r (radial) or e
    (harmonic): the same amortised-density reading as the default."""

    central_band: int = 1
    scale_num: int = 2
    scale_den: int = 1
    decay: str = "radial"


DEFAULT_SPEC = MaskSpec()


def width_and_period(dist, s, spec=DEFAULT_SPEC):
    """(w, c) of one frame distance, in exact integer / rational arithmetic."""
    dist, s = int(dist), int(s)
    cb = spec.central_band
    if dist <= cb:
        return s, 1
    if spec.decay == "harmonic":
        e = dist - cb + 1
        w = s // e
        return w, (1 if w >= 1 else -(-e // s))
    p, q = spec.scale_num, spec.scale_den
    # smallest r >= 1 with dist < (cb+1) (p/q)^r, i.e. dist * q^r < (cb+1) * p^r
    r = 1
    while not (dist * q ** r < (cb + 1) * p ** r):
        r += 1
    w = (s * q ** r) // (p ** r)                      # floor(s / sigma^r)
    c = 1 if w >= 1 else -(-(p ** r) // (s * q ** r))  # ceil(sigma^r / s)
    return w, c


def spec_distance_table(f, s, spec=DEFAULT_SPEC):
    """(h, c) for every frame distance in [0, f) under a mask spec."""
    wc = [width_and_period(d, s, spec) for d in range(max(f, 1))]
    h = np.array([w - 1 for w, _ in wc], dtype=np.int64)
    c = np.array([c for _, c in wc], dtype=np.int64)
    return h, c


# ---------------------------------------------------------------------------
# Token-level mask (Eq.4 + Eq.8, flattened)
# ---------------------------------------------------------------------------

def allowed(i, k, j, l, s, sink=True, spec=None):
    """Allowed(query frame i pos k, key frame j pos l); broadcasts over arrays.

    (sink and j == 0)  or  (h(d) >= 0 and |k-l| <= h(d))
                       or  (h(d) < 0 and d mod c(d) == 0 and k == l),  d = |i-j|.
    spec None: the method's own rule (closed form); a MaskSpec: an ablation.
    """
    i = np.asarray(i, dtype=np.int64)
    j = np.asarray(j, dtype=np.int64)
    k = np.asarray(k, dtype=np.int64)
    l = np.asarray(l, dtype=np.int64)
    d = np.abs(i - j)
    if spec is None:
        h = half_width(d, s)
        c = sample_period(d, s)
    else:
        H, Cp = spec_distance_table(int(d.max()) + 1 if d.size else 1, s, spec)
        h, c = H[d], Cp[d]
    band = (h >= 0) & (np.abs(k - l) <= h)
    sampled = (h < 0) & (d % c == 0) & (k == l)
    out = band | sampled
    if sink:
        out = out | (j == 0)
    return out


def allowed_tokens(a, b, s, sink=True, spec=None):
    """allowed() on flat token indices a (query) and b (key)."""
    a = np.asarray(a, dtype=np.int64)
    b = np.asarray(b, dtype=np.int64)
    return allowed(a // s, a % s, b // s, b % s, s, sink, spec)


def token_mask(f, s, sink=True, spec=None):
    """Dense n x n boolean mask (True = allowed).  Tiny shapes only."""
    n = f * s
    a = np.arange(n, dtype=np.int64)
    return allowed_tokens(a[:, None], a[None, :], s, sink, spec)


def _mask_from_table(qi, qk, kj, kl, f, s, sink, spec=None):
    """allowed() over a (queries x keys) grid using the per-distance table
    (h(d), c(d)) of distance_table() instead of recomputing it per pair.
    Same predicate, int32 arithmetic."""
    H, Cp = distance_table(f, s) if spec is None else spec_distance_table(f, s, spec)
    H = H.astype(np.int32)
    Cp = Cp.astype(np.int32)
    if qi.size and (qi == qi[0]).all():
        # every query in one frame: d, h(d), c(d) depend on the key alone
        d1 = np.abs(qi[0] - kj)
        h1 = H[d1]
        out = np.abs(qk[:, None] - kl[None, :]) <= h1[None, :]      # h < 0 never passes
        samp = (h1 < 0) & (d1 % Cp[d1] == 0)
        if samp.any():
            out[:, samp] |= qk[:, None] == kl[samp][None, :]
        if sink:
            out[:, kj == 0] = True
        return out
    d = np.abs(qi[:, None] - kj[None, :])
    h = H[d]
    out = np.abs(qk[:, None] - kl[None, :]) <= h          # h < 0 never passes
    if (H < 0).any():
        c = Cp[d]
        out |= (h < 0) & (d % c == 0) & (qk[:, None] == kl[None, :])
    if sink:
        out |= (kj == 0)[None, :]
    return out


def row_mask(rows, f, s, sink=True, spec=None):
    """Boolean mask of the given query rows against all n keys."""
    n = f * s
    rows = np.asarray(rows, dtype=np.int32)
    b = np.arange(n, dtype=np.int32)
    return _mask_from_table(rows // s, rows % s, b // s, b % s, f, s, sink, spec)


def col_mask(cols, f, s, sink=True, spec=None):
    """Boolean mask of all n queries against the given key columns (n x len)."""
    n = f * s
    cols = np.asarray(cols, dtype=np.int32)
    a = np.arange(n, dtype=np.int32)
    return _mask_from_table(a // s, a % s, cols // s, cols % s, f, s, sink, spec)


def pair_mask(rows, cols, f, s, sink=True, spec=None):
    """Boolean mask of the given query rows against the given key columns."""
    rows = np.asarray(rows, dtype=np.int32)
    cols = np.asarray(cols, dtype=np.int32)
    return _mask_from_table(rows // s, rows % s, cols // s, cols % s, f, s, sink, spec)


def key_superset(a0, a1, f, s, sink=True, spec=None):
    """Key indices (sorted, int64) that include every key any query row in
    [a0, a1) may attend to.  The rows must lie in one frame i.

    Per key frame j the allowed keys of row (i, k) are, by the rule of
    allowed(): all of frame 0 (sink), the window |k - l| <= h(d), the single
    position l = k (sampled diagonal, on its period), or nothing.  Over
    k in [k0, k1] their union lies inside [k0 - h, k1 + h] (or [k0, k1]),
    clipped to the frame; those ranges are returned.  Used to skip keys whose
    logits are masked for every row of a chunk -- they would only add
    exp(-inf) = 0 to each sum -- when the oracle evaluates whole heads."""
    i = a0 // s
    assert 0 <= a0 < a1 <= (i + 1) * s, "rows must lie in one frame"
    k0, k1 = a0 - i * s, a1 - 1 - i * s
    H, Cp = distance_table(f, s) if spec is None else spec_distance_table(f, s, spec)
    parts = []
    for j in range(f):
        d = abs(i - j)
        h, c = int(H[d]), int(Cp[d])
        if sink and j == 0:
            lo, hi = 0, s - 1
        elif h >= 0:
            lo, hi = max(0, k0 - h), min(s - 1, k1 + h)
        elif d % c == 0:
            lo, hi = k0, k1
        else:
            continue
        parts.append(np.arange(j * s + lo, j * s + hi + 1, dtype=np.int64))
    return np.concatenate(parts) if parts else np.zeros(0, dtype=np.int64)


# ---------------------------------------------------------------------------
# Block tiles: brute force
# ---------------------------------------------------------------------------

def tile_states_bruteforce(f, s, B, sink=True, spec=None):
    """uint8 [nb, nb]: 0 inactive, TILE_FULL, TILE_PARTIAL -- from the token mask."""
    n = f * s
    nb = -(-n // B)
    m = np.zeros((nb * B, nb * B), dtype=bool)
    m[:n, :n] = token_mask(f, s, sink, spec)
    t = m.reshape(nb, B, nb, B)
    active = t.any(axis=(1, 3))
    every = t.all(axis=(1, 3))
    inside = (np.arange(nb) + 1) * B <= n
    full = every & inside[:, None] & inside[None, :]
    out = np.zeros((nb, nb), dtype=np.uint8)
    out[active] = TILE_PARTIAL
    out[full] = TILE_FULL
    return out


# ---------------------------------------------------------------------------
# Block tiles: frame-segment interval test (scales to n ~ 5e5)
# ---------------------------------------------------------------------------

def _segments(nb, B, n, s):
    """Per block: its in-range tokens split by frame -> (frame, lo, hi) arrays
    of shape [nb, S] plus a validity mask (positions are inclusive)."""
    S = (B + s - 1) // s + 1          # max frames a block can touch
    start = np.arange(nb, dtype=np.int64) * B
    stop = np.minimum(start + B, n)     # exclusive
    frame = np.zeros((nb, S), dtype=np.int64)
    lo = np.zeros((nb, S), dtype=np.int64)
    hi = np.zeros((nb, S), dtype=np.int64)
    valid = np.zeros((nb, S), dtype=bool)
    f0 = start // s
    for t in range(S):
        fr = f0 + t
        a0 = np.maximum(start, fr * s)
        a1 = np.minimum(stop, (fr + 1) * s)   # exclusive
        ok = a0 < a1
        frame[:, t] = fr
        lo[:, t] = a0 - fr * s
        hi[:, t] = a1 - 1 - fr * s
        valid[:, t] = ok
    return frame, lo, hi, valid


def tile_states_intervals(f, s, B, sink=True, chunk=64, spec=None):
    """uint8 [nb, nb] tile states from the interval test.

    For a query segment (frame i, positions [k0, k1]) and a key segment
    (frame j, positions [l0, l1]) with d = |i - j|:
      sink and j == 0        -> every pair allowed;
      h(d) >= 0              -> some pair iff gap <= h, every pair iff span <= h,
                                gap = max(0, l0-k1, k0-l1), span = max(k1-l0, l1-k0);
      h(d) < 0, d%c(d) == 0  -> some pair iff the intervals intersect, every pair
                                iff both are the same single position;
      otherwise              -> no pair.
    """
    n = f * s
    nb = -(-n // B)
    fr, lo, hi, va = _segments(nb, B, n, s)
    inside = (np.arange(nb) + 1) * B <= n
    if spec is not None:
        Ht, Ct = spec_distance_table(f, s, spec)
    out = np.zeros((nb, nb), dtype=np.uint8)
    # key-side arrays broadcast as [1, 1, nb, S]
    jf, l0, l1, jv = (x[None, None] for x in (fr, lo, hi, va))
    for q0 in range(0, nb, chunk):
        q1 = min(nb, q0 + chunk)
        i_, k0, k1, iv = (x[q0:q1, :, None, None] for x in (fr, lo, hi, va))
        d = np.abs(i_ - jf)
        if spec is None:
            h = half_width(d, s)
            c = sample_period(d, s)
        else:
            dd = np.minimum(d, f - 1)      # distances >= f only occur on invalid segments
            h, c = Ht[dd], Ct[dd]
        gap = np.maximum(0, np.maximum(l0 - k1, k0 - l1))
        span = np.maximum(k1 - l0, l1 - k0)
        band_any = (h >= 0) & (gap <= h)
        band_all = (h >= 0) & (span <= h)
        on_period = (h < 0) & (d % c == 0)
        samp_any = on_period & (gap == 0)
        samp_all = on_period & (k0 == k1) & (l0 == l1) & (k0 == l0)
        any_ = band_any | samp_any
        all_ = band_all | samp_all
        if sink:
            any_ = any_ | (jf == 0)
            all_ = all_ | (jf == 0)
        pair = iv & jv
        any_tile = (any_ & pair).any(axis=(1, 3))
        # every valid segment pair must be all-allowed; invalid pairs are neutral
        all_tile = (all_ | ~pair).all(axis=(1, 3))
        full = all_tile & inside[q0:q1, None] & inside[None, :]
        blk = np.zeros(any_tile.shape, dtype=np.uint8)
        blk[any_tile] = TILE_PARTIAL
        blk[any_tile & full] = TILE_FULL
        out[q0:q1] = blk
    return out


# ---------------------------------------------------------------------------
# CSR / CSC / longest-row-first order
# ---------------------------------------------------------------------------

def csr_from_states(st):
    """Row-major CSR of the active tiles: (row_ptr, col_idx ascending, kind)."""
    nb = st.shape[0]
    active = st != 0
    counts = active.sum(axis=1)
    row_ptr = np.zeros(nb + 1, dtype=np.int32)
    row_ptr[1:] = np.cumsum(counts)
    r, c = np.nonzero(active)              # row-major, columns ascending
    return row_ptr, c.astype(np.int32), st[r, c].astype(np.uint8)


def csc_from_states(st):
    """Column-major CSC: (col_ptr, row_idx ascending, kind)."""
    return csr_from_states(np.ascontiguousarray(st.T))


def row_order(row_ptr):
    """Rows by active-tile count descending, ties by row index ascending."""
    counts = np.diff(np.asarray(row_ptr, dtype=np.int64))
    idx = np.arange(counts.size)
    return np.lexsort((idx, -counts)).astype(np.int32)


def block_csr(f, s, B, sink=True, method="intervals", spec=None):
    """Everything the block-sparse executor needs, as a dict of numpy arrays."""
    if method == "bruteforce":
        st = tile_states_bruteforce(f, s, B, sink, spec)
    else:
        st = tile_states_intervals(f, s, B, sink, spec=spec)
    row_ptr, col_idx, kind = csr_from_states(st)
    col_ptr, row_idx, kind_t = csc_from_states(st)
    return dict(
        n_blocks=st.shape[0], states=st,
        row_ptr=row_ptr, col_idx=col_idx, kind=kind,
        col_ptr=col_ptr, row_idx=row_idx, kind_t=kind_t,
        row_order=row_order(row_ptr), col_order=row_order(col_ptr),
    )


# ---------------------------------------------------------------------------
# Pair counting (complexity invariants, [review] §4.2 Eq.5/Eq.6)
# ---------------------------------------------------------------------------

def allowed_pair_count(f, s, sink=True, spec=None):
    """Number of allowed (query, key) token pairs, summed per frame pair.

    Counts positions directly per frame pair: for each (i, j) build the s x s
    block from allowed() and count it.  O(f^2 s^2) -- small shapes only.
    """
    k = np.arange(s)[:, None]
    l = np.arange(s)[None, :]
    total = 0
    for i in range(f):
        for j in range(f):
            total += int(allowed(i, k, j, l, s, sink, spec).sum())
    return total
