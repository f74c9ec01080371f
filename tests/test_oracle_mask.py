"""Pins of the CPU reference mask to what the pages and the mathematics fix.

Sources: the worked toy example and §4.2 of the Radial Attention review
(jaehun.me); the central-band / constant-sparsity statements of the authors'
responses (paperhub.cn).  None of these tests re-types the oracle's formula:
they check printed values, brute force, closed-form counts and invariants.
"""

import math
import os

import numpy as np
import pytest

from oracle import mask as M


def _load_toy(golden_dir):
    spec = {"width": {}, "keys": {}}
    with open(os.path.join(golden_dir, "toy_example.txt")) as fh:
        for line in fh:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            tok = line.split()
            if tok[0] in ("f", "s", "i0", "k0"):
                spec[tok[0]] = int(tok[1])
            elif tok[0] == "width":
                spec["width"][int(tok[1])] = int(tok[2])
            elif tok[0] == "keys":
                spec["keys"][(int(tok[1]), int(tok[2]))] = {int(x) for x in tok[3].split(",")}
    return spec


def _toy_matches(spec, allowed_fn):
    f, s, i0, k0 = spec["f"], spec["s"], spec["i0"], spec["k0"]
    for (sink, j), want in spec["keys"].items():
        got = {l for l in range(s) if bool(allowed_fn(i0, k0, j, l, s, bool(sink)))}
        if got != want:
            return False
    return True


def test_toy_example_widths(golden_dir):
    spec = _load_toy(golden_dir)
    for j, w in spec["width"].items():
        assert int(M.diag_width(abs(spec["i0"] - j), spec["s"])) == w


def test_toy_example_key_sets(golden_dir):
    spec = _load_toy(golden_dir)
    assert _toy_matches(spec, M.allowed)


def test_toy_example_catches_planted_width_mistake(golden_dir):
    """Keeping |k-l| <= w (the 'half-width taken literally' misreading) keeps
    l = 0..8 in frame 0 and must fail the printed l = 1..7."""
    spec = _load_toy(golden_dir)

    def wrong(i, k, j, l, s, sink):
        d = abs(i - j)
        w = int(M.diag_width(d, s))
        return (sink and j == 0) or abs(k - l) <= w

    assert not _toy_matches(spec, wrong)


GRIDS = [
    # (f, s, B): B > s, B not dividing s, B dividing s, sampling branch, f <= 2
    (4, 9, 4), (4, 9, 16), (8, 16, 16), (8, 16, 64), (6, 10, 8), (5, 7, 3),
    (16, 8, 8), (64, 4, 16), (40, 3, 8), (33, 5, 16), (2, 13, 8), (1, 20, 8),
    (12, 24, 32), (9, 30, 64), (20, 6, 128),
]


@pytest.mark.parametrize("f,s,B", GRIDS)
@pytest.mark.parametrize("sink", [True, False])
def test_interval_tiles_equal_bruteforce(f, s, B, sink):
    a = M.tile_states_bruteforce(f, s, B, sink)
    b = M.tile_states_intervals(f, s, B, sink)
    np.testing.assert_array_equal(a, b)


def test_interval_tiles_random_grids():
    rng = np.random.default_rng(1234)
    for _ in range(40):
        f = int(rng.integers(1, 40))
        s = int(rng.integers(1, 40))
        B = int(rng.choice([2, 4, 8, 16, 32, 64]))
        sink = bool(rng.integers(0, 2))
        if f * s > 1500:
            continue
        np.testing.assert_array_equal(M.tile_states_bruteforce(f, s, B, sink),
                                      M.tile_states_intervals(f, s, B, sink))


@pytest.mark.parametrize("f,s", [(8, 16), (5, 9), (64, 4), (17, 6)])
def test_same_frame_is_dense(f, s):
    m = M.token_mask(f, s, sink=False)
    for i in range(f):
        assert m[i * s:(i + 1) * s, i * s:(i + 1) * s].all()


def test_half_width_non_increasing_and_central_band_dense():
    for s in (1, 3, 9, 64, 1560, 3600):
        h, _ = M.distance_table(300, s)
        assert h[0] == s - 1 and h[1] == s - 1       # |i-j| <= 1 dense
        assert np.all(np.diff(h) <= 0)


def test_width_halves_per_band():
    """Fig.5: density halves from one temporal band to the next."""
    s = 1024
    for d in range(2, 200):
        r = int(math.floor(math.log2(d)))
        assert M.diag_width(d, s) == s >> r


@pytest.mark.parametrize("f,s", [(8, 16), (16, 4), (9, 7)])
def test_symmetric_without_sink(f, s):
    m = M.token_mask(f, s, sink=False)
    assert (m == m.T).all()


def test_sink_breaks_symmetry_and_reaches_frame0():
    f, s = 8, 16
    m = M.token_mask(f, s, sink=True)
    assert m[:, :s].all()                     # every query sees frame 0
    assert not (m == m.T).all()


@pytest.mark.parametrize("s", [1, 5, 16])
def test_two_frames_or_fewer_is_all_ones(s):
    for f in (1, 2):
        assert M.token_mask(f, s, sink=False).all()


def _lattice_band_count(s, h):
    """#{(k, l) in [0,s)^2 : |k-l| <= h}: count the diagonals directly."""
    h = min(h, s - 1)
    return sum(s - abs(t) for t in range(-h, h + 1))


@pytest.mark.parametrize("f,s", [(16, 8), (12, 13), (64, 4), (33, 9)])
def test_pair_count_per_frame_pair(f, s):
    """Frame-pair block counts equal the band lattice count s(2h+1)-h(h+1)
    (h >= 0) or s / 0 (sampled diagonal), and the diagonal sum agrees."""
    m = M.token_mask(f, s, sink=False)
    for i in range(f):
        for j in range(f):
            d = abs(i - j)
            h = int(M.half_width(d, s))
            got = int(m[i * s:(i + 1) * s, j * s:(j + 1) * s].sum())
            if h >= 0:
                hh = min(h, s - 1)
                assert got == s * (2 * hh + 1) - hh * (hh + 1) == _lattice_band_count(s, hh)
            else:
                c = int(M.sample_period(d, s))
                assert got == (s if d % c == 0 else 0)


def test_pair_count_helper_matches_token_mask():
    for f, s, sink in [(8, 16, True), (9, 5, False), (64, 4, True)]:
        assert M.allowed_pair_count(f, s, sink) == int(M.token_mask(f, s, sink).sum())


def test_n_log_n_bound():
    """[review] §4.2 Eq.5/6: O(n log n) for fixed s.  Band r >= 1 covers 2^r
    frame distances, each with <= 2f ordered frame pairs of <= s(2h+1) <= 2s^2/2^r
    allowed pairs, so <= 4fs^2 = 4ns per band and there are <= log2 f such
    bands; band 0 (distances 0, 1) holds <= 3ns; the sink adds <= ns.
    Hence pairs <= n s (4 + 4 log2 f)."""
    s = 8
    ratios = []
    for f in (2, 4, 8, 16, 32, 64, 128):
        n = f * s
        pairs = M.allowed_pair_count(f, s, sink=True)
        assert pairs <= n * s * (4 + 4 * math.log2(f))
        ratios.append(pairs / (n * math.log2(n)))
    # bounded, not growing like n: the ratio at f=128 stays below 2x its f=16 value
    assert ratios[-1] < 2 * ratios[3]
    # while dense growth would be n / log n: quadratic count grows ~x16 from f=32 to 128
    assert M.allowed_pair_count(128, s, True) < 16 * M.allowed_pair_count(32, s, True) / 2


def test_density_constant_across_resolution():
    """[rebuttal]: sparsity stays constant across resolutions for fixed f.
    Per frame pair the count is s^2 (2/2^r - 1/4^r) + O(s), so densities at two
    resolutions differ by at most ~8/s each (derivation in the test module)."""
    f = 16
    dens = {}
    for s in (64, 128, 256):
        dens[s] = M.allowed_pair_count(f, s, sink=False) / float((f * s) ** 2)
    for a in dens:
        for b in dens:
            assert abs(dens[a] - dens[b]) <= 8.0 / a + 8.0 / b


def test_tail_tiles_never_full_and_rows_nonempty():
    for f, s, B in [(3, 10, 8), (5, 9, 4), (7, 13, 16)]:
        st = M.tile_states_intervals(f, s, B, True)
        n = f * s
        nb = st.shape[0]
        if n % B:
            assert (st[-1] != M.TILE_FULL).all() and (st[:, -1] != M.TILE_FULL).all()
        assert (st != 0).any(axis=1).all()       # every row has a tile (diagonal)
        assert all(st[t, t] != 0 for t in range(nb))


def test_csr_csc_roundtrip_and_order():
    f, s, B = 9, 30, 16
    c = M.block_csr(f, s, B, True)
    st = c["states"]
    nb = c["n_blocks"]
    dense = np.zeros_like(st)
    for r in range(nb):
        for p in range(c["row_ptr"][r], c["row_ptr"][r + 1]):
            dense[r, c["col_idx"][p]] = c["kind"][p]
        cols = c["col_idx"][c["row_ptr"][r]:c["row_ptr"][r + 1]]
        assert np.all(np.diff(cols) > 0)
    np.testing.assert_array_equal(dense, st)
    denseT = np.zeros_like(st)
    for q in range(nb):
        for p in range(c["col_ptr"][q], c["col_ptr"][q + 1]):
            denseT[c["row_idx"][p], q] = c["kind_t"][p]
    np.testing.assert_array_equal(denseT, st)
    cnt = np.diff(c["row_ptr"])
    o = c["row_order"]
    assert sorted(o.tolist()) == list(range(nb))
    for a, b in zip(o[:-1], o[1:]):
        assert cnt[a] > cnt[b] or (cnt[a] == cnt[b] and a < b)


def test_sampling_branch_reached_on_tiny_grid():
    """f=64, s=4: w(d) = 0 from d = 8 on, so the sampled diagonal is used."""
    f, s = 64, 4
    h, c = M.distance_table(f, s)
    assert (h[8:] < 0).all() and (h[:8] >= 0).all()
    m = M.token_mask(f, s, sink=False)
    # frame distance 8: c = 2 -> kept (8 % 2 == 0), diagonal only
    blk = m[0:s, 8 * s:9 * s]
    assert (blk == np.eye(s, dtype=bool)).all()
    # frame distance 9: c = 2 -> not on the period -> nothing
    assert not m[0:s, 9 * s:10 * s].any()


def _band_sums(f, s):
    """Kept pairs per temporal band, counted on the brute-force token mask
    (sink off): B(r) = sum over the band's distances d in [2^r, 2^(r+1)) of
    the allowed (k, l) pairs between frame 0 and frame d."""
    m = M.token_mask(f, s, sink=False)
    per_d = np.array([int(m[0:s, d * s:(d + 1) * s].sum()) for d in range(f)])
    sums = {}
    r = 1
    while 2 ** (r + 1) <= f:
        sums[r] = int(per_d[2 ** r:2 ** (r + 1)].sum())
        r += 1
    return per_d, sums


@pytest.mark.parametrize("f,s", [(256, 4), (256, 3), (512, 5), (128, 2)])
def test_sampled_diagonal_keeps_the_amortised_density_decay(f, s):
    """[review] Fig.5 caption and [rebuttal] (diagonal frequency reduction):
    once a band's diagonal width falls below one token, frame pairs are
    subsampled so that the AMORTISED density keeps decaying as before, i.e.
    it keeps halving from one temporal band to the next, and what is kept is
    the main diagonal only.  Counted by brute force, independent of the rule
    that produces it: the band's density rho(r) = B(r) / (2^r s^2) must halve
    per band (ratio within [1/3, 1] once ceil rounding is allowed for), and
    the kept pairs per band, B(r) = rho(r) 2^r s^2, stay between 3/4 and 2
    times those of the last band whose width is still one token (that band
    holds 2^r s pairs with s/2 < 2^r <= s; a halving density keeps B(r) near
    s^2 from then on).  A rule that keeps the
    diagonal in every pair (density stops falling), in no pair, or subsampled
    by 2^r instead of 2^r / s (density falls s times too fast) fails here."""
    per_d, sums = _band_sums(f, s)
    widths = {r: s // 2 ** r for r in sums}
    sampled = [r for r in sums if widths[r] == 0]
    last_w1 = max(r for r in sums if widths[r] == 1)
    assert len(sampled) >= 3, "grid too small to reach several sampled bands"
    rho = {r: sums[r] / (2 ** r * s * s) for r in sums}
    for r in [last_w1] + sampled:
        if r - 1 in rho and widths[r - 1] <= 1:
            ratio = rho[r] / rho[r - 1]
            assert 1.0 / 3.0 <= ratio <= 1.0, (r, ratio)
    for r in sampled:
        assert 0.75 * sums[last_w1] <= sums[r] <= 2 * sums[last_w1], (r, sums[r], sums[last_w1])
    # the pages describe diagonal samples: in a sampled band a kept frame pair
    # holds the main diagonal k == l and nothing else
    m = M.token_mask(f, s, sink=False)
    for r in sampled:
        for d in range(2 ** r, 2 ** (r + 1)):
            blk = m[0:s, d * s:(d + 1) * s]
            assert (not blk.any()) or (blk == np.eye(s, dtype=bool)).all(), d
    # and the total still grows like n log n: band sums do not grow with r
    assert max(sums[r] for r in sampled) <= 2 * s * s


@pytest.mark.parametrize("f,s,sink", [(8, 16, True), (64, 4, False), (64, 4, True), (9, 7, True), (1, 5, False)])
def test_row_and_col_masks_equal_token_mask(f, s, sink):
    full = M.token_mask(f, s, sink)
    n = f * s
    rows = np.arange(0, n, 3)
    np.testing.assert_array_equal(M.row_mask(rows, f, s, sink), full[rows])
    np.testing.assert_array_equal(M.col_mask(rows, f, s, sink), full[:, rows])
