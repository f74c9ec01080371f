"""Ablation masks on the device (central-band width, width scale between
bands, harmonic decay): the block CSR must be bit-exact with the CPU
reference, and attention under them must match it within the tolerances of
the default-mask tests."""

import numpy as np
import pytest
import torch

import block_sparse_attention_csr_b200 as rb
from block_sparse_attention_csr_b200 import inputs as I
from oracle import attention as A
from oracle import mask as M

pytestmark = pytest.mark.gpu

VARIANTS = [
    # (central_band, (num, den), decay)
    (0, (2, 1), "radial"),
    (2, (2, 1), "radial"),
    (1, (3, 2), "radial"),
    (1, (3, 1), "radial"),
    (1, (4, 1), "radial"),
    (1, (2, 1), "harmonic"),
    (2, (3, 2), "harmonic"),
]


def _spec(cb, ws, decay):
    return M.MaskSpec(central_band=cb, scale_num=ws[0], scale_den=ws[1], decay=decay)


@pytest.mark.parametrize("cb,ws,decay", VARIANTS)
@pytest.mark.parametrize("f,s,B,sink", [(33, 3600, 128, 1), (21, 1560, 128, 0), (64, 4, 64, 1), (40, 3, 128, 1),
                                        (9, 1000, 64, 1)])
def test_variant_csr_bit_exact(cb, ws, decay, f, s, B, sink):
    csr = rb.radial_mask_build(f, s, B, sink=sink, central_band=cb, width_scale=ws, decay=decay)
    got = rb.radial_csr_copy_to_host(csr)
    ref = M.block_csr(f, s, B, bool(sink), spec=_spec(cb, ws, decay))
    for key in ("row_ptr", "col_idx", "kind", "col_ptr", "row_idx", "kind_t", "row_order", "col_order"):
        np.testing.assert_array_equal(got[key], ref[key], err_msg=key)


@pytest.mark.parametrize("cb,ws,decay", VARIANTS)
def test_variant_attention_parity(cb, ws, decay):
    f, s, block = 12, 300, 128
    wl = I.small_workload("var", 1, 2, 128, f, s, block, seed=61)
    q, k, v, do = I.draw(wl, device="cuda", backward=True)
    csr = rb.radial_mask_build(f, s, block, sink=1, central_band=cb, width_scale=ws, decay=decay)
    o, lse = rb.radial_attn_fwd(csr, q, k, v)
    dq, dk, dv = rb.radial_attn_bwd(csr, do, q, k, v, o, lse)
    rb.radial_device_status()
    spec = _spec(cb, ws, decay)
    x = [t.float().cpu().numpy() for t in (q, k, v, do)]
    o_ref, l_ref = A.radial_forward(x[0], x[1], x[2], f, s, True, spec=spec)
    err = np.abs(o.float().cpu().numpy() - o_ref)
    assert err.max() <= 2e-2 and err.mean() <= 2e-3
    assert np.abs(lse.cpu().numpy() - l_ref).max() <= 1e-3
    g_ref = A.radial_backward(x[0], x[1], x[2], o_ref, x[3], l_ref, f, s, True, spec=spec)
    for g, r in zip((dq, dk, dv), g_ref):
        assert np.abs(g.float().cpu().numpy() - r).max() <= 5e-2
