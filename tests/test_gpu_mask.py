"""Device mask builder vs the CPU reference: block CSR, CSC and orders must be
bit-exact (index work)."""

import numpy as np
import pytest

import block_sparse_attention_csr_b200 as rb
from oracle import mask as M

pytestmark = pytest.mark.gpu

SHAPES = [
    # (frames, tokens_per_frame, block, sink): tiny config, benchmark shapes,
    # sweep, blocks not aligned to frames, s < block, sampling branch, f <= 2
    (8, 64, 64, 1),
    (21, 1560, 128, 1),
    (33, 3600, 128, 1),
    (132, 3600, 128, 1),
    (8, 3600, 128, 1), (16, 3600, 128, 1), (66, 3600, 128, 1),
    (32, 256, 64, 1), (32, 256, 64, 0),
    (33, 3600, 128, 0),
    (5, 200, 128, 1), (7, 300, 64, 0),
    (40, 3, 128, 1), (64, 4, 64, 0), (64, 4, 64, 1), (200, 5, 128, 0),
    (1, 1, 64, 1), (1, 1000, 128, 1), (2, 77, 64, 0), (3, 129, 128, 1),
]


def _compare(c_dev, ref):
    np.testing.assert_array_equal(c_dev["row_ptr"], ref["row_ptr"])
    np.testing.assert_array_equal(c_dev["col_idx"], ref["col_idx"])
    np.testing.assert_array_equal(c_dev["kind"], ref["kind"])
    np.testing.assert_array_equal(c_dev["col_ptr"], ref["col_ptr"])
    np.testing.assert_array_equal(c_dev["row_idx"], ref["row_idx"])
    np.testing.assert_array_equal(c_dev["kind_t"], ref["kind_t"])
    np.testing.assert_array_equal(c_dev["row_order"], ref["row_order"])
    np.testing.assert_array_equal(c_dev["col_order"], ref["col_order"])


@pytest.mark.parametrize("f,s,B,sink", SHAPES)
def test_mask_csr_bit_exact(f, s, B, sink):
    csr = rb.radial_mask_build(f, s, B, sink=sink)
    info = rb.radial_csr_info(csr)
    ref = M.block_csr(f, s, B, bool(sink))
    assert info["n_blocks"] == ref["n_blocks"]
    assert info["nnz"] == len(ref["col_idx"])
    assert info["n_full"] == int((ref["kind"] == M.TILE_FULL).sum())
    _compare(rb.radial_csr_copy_to_host(csr), ref)


@pytest.mark.parametrize("n,B", [(1, 64), (1000, 128), (4096, 64), (118800, 128)])
def test_dense_csr(n, B):
    csr = rb.radial_mask_build_dense(n, B)
    ref = M.block_csr(1, n, B, False)
    _compare(rb.radial_csr_copy_to_host(csr), ref)
    nb = -(-n // B)
    assert rb.radial_csr_info(csr)["nnz"] == nb * nb


def test_random_small_grids():
    rng = np.random.default_rng(7)
    for _ in range(25):
        f, s = int(rng.integers(1, 60)), int(rng.integers(1, 300))
        B = int(rng.choice([64, 128]))
        sink = int(rng.integers(0, 2))
        csr = rb.radial_mask_build(f, s, B, sink=sink)
        _compare(rb.radial_csr_copy_to_host(csr), M.block_csr(f, s, B, bool(sink)))
