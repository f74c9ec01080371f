"""The benchmark's closed-form pair count against the oracle's brute force.

`bench.allowed_pairs` feeds the element-level throughput of the bench line
(4*d flops per allowed pair).  The oracle counts allowed pairs position by
position from its token rule ([review] §4.2, Eq.4, Fig.5; sink App. A.1 Eq.8).
"""
import pytest

import bench
from oracle.mask import allowed_pair_count


@pytest.mark.parametrize("f,s,sink", [
    (5, 7, True),     # bands wider than the frame at d <= 1, clipped bands beyond
    (8, 64, True),    # several bands
    (6, 33, False),   # sink off
    (64, 4, False),   # sampled diagonals (width < 1) at large distances
    (40, 3, True),    # s < 4: most distances sampled, sink on
    (3, 1, True),     # one token per frame
    (12, 20, False),
])
def test_allowed_pairs_matches_oracle(f, s, sink):
    assert bench.allowed_pairs(f, s, sink) == allowed_pair_count(f, s, sink)


def test_hunyuan_element_flops():
    """The HunyuanVideo shape's 67.84 element-TFLOP per forward launch."""
    from block_sparse_attention_csr_b200 import inputs as I
    wl = I.WORKLOADS["hunyuan720p"]
    pairs = bench.allowed_pairs(wl.frames, wl.tokens_per_frame)
    assert abs(bench.elem_flops(wl, pairs) / 1e12 - 67.84) < 0.01


def test_hunyuan_tile_flops_from_oracle_plan():
    """Tile-level work of the bench line: 4*B^2*d flops per active 128x128 tile
    (QK^T and PV) over the oracle's own tile classification -- 389,411 active
    tiles per head and 78.40 TFLOP per forward launch at the HunyuanVideo shape."""
    import numpy as np
    from block_sparse_attention_csr_b200 import inputs as I
    from oracle.mask import tile_states_intervals
    wl = I.WORKLOADS["hunyuan720p"]
    nnz = int(np.count_nonzero(tile_states_intervals(wl.frames, wl.tokens_per_frame, wl.block, True)))
    assert nnz == 389_411
    assert abs(bench.tile_flops(wl, nnz) / 1e12 - 78.40) < 0.01
