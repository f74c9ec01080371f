"""Radial Attention's block-sparse masked attention on B200 (sm_100a).

The hot path lives in ``libradial.so`` (CUDA kernels behind the C ABI of
``include/radial.h``); this package is its thin Python binding plus the seeded
synthetic workload generators.  Nothing here computes attention on the host,
and there is no fallback: calls raise if the library is missing.
"""

from ._binding import (  # noqa: F401
    Csr,
    RadialError,
    lib_path,
    load,
    make_desc,
    radial_attn_bwd,
    radial_attn_bwd_noalloc,
    radial_attn_bwd_workspace_size,
    radial_attn_fwd,
    radial_attn_fwd_staged,
    radial_csr_copy_to_host,
    radial_csr_info,
    radial_device_status,
    radial_launch_count,
    radial_lora_bwd,
    radial_lora_fwd,
    radial_mask_build,
    radial_mask_build_dense,
    radial_params_default,
    radial_selftest_bounded_wait,
)

TILE_FULL = 1
TILE_PARTIAL = 2
