"""Pins of the CPU reference's ablation masks: the central-band width and the
width scale between bands of the authors' responses (paperhub.cn), and the
harmonic-series decay of the review's App. C.3.  The default spec must give
back the method's own closed form; each variant is checked against the
property that defines it and against brute-force tiles."""

import math

import numpy as np
import pytest

from oracle import mask as M

SPECS = [
    M.MaskSpec(),                                   # the method's default
    M.MaskSpec(central_band=0),
    M.MaskSpec(central_band=2),
    M.MaskSpec(scale_num=3, scale_den=2),           # width scale 1.5
    M.MaskSpec(scale_num=3),
    M.MaskSpec(scale_num=4),
    M.MaskSpec(decay="harmonic"),
    M.MaskSpec(central_band=2, decay="harmonic"),
]


@pytest.mark.parametrize("s", [1, 3, 9, 64, 100, 1560, 3600])
def test_default_spec_is_the_closed_form(s):
    h_closed, c_closed = M.distance_table(600, s)
    h_spec, c_spec = M.spec_distance_table(600, s, M.DEFAULT_SPEC)
    np.testing.assert_array_equal(h_closed, h_spec)
    np.testing.assert_array_equal(c_closed[h_closed < 0], c_spec[h_spec < 0])


@pytest.mark.parametrize("cb", [0, 1, 2, 3])
def test_central_band_is_dense_exactly_up_to_its_width(cb):
    s = 64
    h, _ = M.spec_distance_table(50, s, M.MaskSpec(central_band=cb))
    assert (h[:cb + 1] == s - 1).all()
    assert h[cb + 1] < s - 1


@pytest.mark.parametrize("num,den", [(2, 1), (3, 2), (3, 1), (4, 1)])
@pytest.mark.parametrize("cb", [0, 1, 2])
def test_width_scale_bands(num, den, cb):
    """Band r >= 1 starts at distance (cb+1) sigma^(r-1) and has width
    floor(s / sigma^r): consecutive bands differ in width by the factor sigma."""
    s = 4096
    sigma = num / den
    spec = M.MaskSpec(central_band=cb, scale_num=num, scale_den=den)
    for d in range(cb + 1, 400):
        w, _ = M.width_and_period(d, s, spec)
        r = 1
        while not (d < (cb + 1) * sigma ** r - 1e-9):
            r += 1
        assert (cb + 1) * sigma ** (r - 1) <= d + 1e-9
        assert w == math.floor(s / sigma ** r + 1e-9)


def test_harmonic_width_is_inverse_to_distance():
    s = 1000
    for cb in (0, 1, 2):
        spec = M.MaskSpec(central_band=cb, decay="harmonic")
        for d in range(cb + 1, 3000):
            w, c = M.width_and_period(d, s, spec)
            e = d - cb + 1
            assert w * e <= s < (w + 1) * e
            if w == 0:
                assert c == -(-e // s)


@pytest.mark.parametrize("spec", SPECS, ids=lambda x: f"{x.decay}-cb{x.central_band}-{x.scale_num}/{x.scale_den}")
@pytest.mark.parametrize("f,s,B,sink", [(9, 16, 16, True), (12, 10, 8, False), (40, 3, 8, True), (6, 50, 32, True)])
def test_variant_interval_tiles_equal_bruteforce(spec, f, s, B, sink):
    np.testing.assert_array_equal(M.tile_states_bruteforce(f, s, B, sink, spec),
                                  M.tile_states_intervals(f, s, B, sink, spec=spec))


@pytest.mark.parametrize("spec", SPECS, ids=lambda x: f"{x.decay}-cb{x.central_band}-{x.scale_num}/{x.scale_den}")
def test_variant_masks_agree_across_routes(spec):
    f, s = 24, 6
    full = M.token_mask(f, s, True, spec)
    rows = np.arange(0, f * s, 5)
    np.testing.assert_array_equal(M.row_mask(rows, f, s, True, spec), full[rows])
    np.testing.assert_array_equal(M.col_mask(rows, f, s, True, spec), full[:, rows])
    # same-frame always dense; symmetric without the sink
    for i in range(f):
        assert full[i * s:(i + 1) * s, i * s:(i + 1) * s].all()
    ns = M.token_mask(f, s, False, spec)
    assert (ns == ns.T).all()


@pytest.mark.parametrize("spec", SPECS, ids=lambda x: f"{x.decay}-cb{x.central_band}-{x.scale_num}/{x.scale_den}")
def test_variants_stay_n_log_n(spec):
    """Every variant keeps the attention pairs within n s (c0 + c1 log2 f):
    per band (or, harmonic, per distance) the kept pairs shrink like the
    width, so the sum over distances grows logarithmically."""
    s = 8
    vals = []
    for f in (16, 32, 64, 128):
        n = f * s
        vals.append(M.allowed_pair_count(f, s, False, spec) / (n * s * (1 + math.log2(f))))
    assert max(vals) < 3 * (spec.central_band + 2)
    assert vals[-1] <= 1.6 * vals[0]
