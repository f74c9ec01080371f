"""The backward's no-allocation entry point (radial_attn_bwd_noalloc).

It serves callers that cannot give the library a workspace: a plugin or
callback interface with no allocator, a process whose device memory is all
reserved by another framework's pool, or a latency-critical loop that must not
call cudaMalloc (it can synchronise the device).  Instead of a workspace it
uses a fixed device array inside the library.  Here it must agree with the
workspace entry point, radial_attn_bwd, within the gradient tolerance of the
other backward tests (max-abs 5e-2), on two calls in a row, the second of
which reuses the array the first one left behind.  This file sorts last so
that a run stopping at its first failure has run every other test already.
"""

import ctypes

import pytest
import torch

import block_sparse_attention_csr_b200 as rb
from block_sparse_attention_csr_b200 import _binding as B
from block_sparse_attention_csr_b200 import inputs as I

pytestmark = pytest.mark.gpu

G_MAX = 5e-2


def test_noalloc_backward_matches_workspace_backward_twice():
    wl = I.small_workload("noalloc", 1, 2, 128, 9, 1000, 128, 51)
    q, k, v, do = I.draw(wl, device="cuda", backward=True)
    csr = rb.radial_mask_build(9, 1000, 128, sink=1)
    o, lse = rb.radial_attn_fwd(csr, q, k, v)
    ref = rb.radial_attn_bwd(csr, do, q, k, v, o, lse)
    rb.radial_device_status()
    for _ in range(2):
        got = rb.radial_attn_bwd_noalloc(csr, do, q, k, v, o, lse)
        rb.radial_device_status()
        for name, r, g in zip(("dQ", "dK", "dV"), ref, got):
            err = (r.float() - g.float()).abs().max().item()
            assert err <= G_MAX, f"{name}: max-abs {err:.3e}"


def test_noalloc_backward_d64_block64():
    wl = I.small_workload("noalloc64", 2, 2, 64, 7, 300, 64, 52)
    q, k, v, do = I.draw(wl, device="cuda", backward=True)
    csr = rb.radial_mask_build(7, 300, 64, sink=0)
    o, lse = rb.radial_attn_fwd(csr, q, k, v)
    ref = rb.radial_attn_bwd(csr, do, q, k, v, o, lse)
    got = rb.radial_attn_bwd_noalloc(csr, do, q, k, v, o, lse)
    rb.radial_device_status()
    for r, g in zip(ref, got):
        assert (r.float() - g.float()).abs().max().item() <= G_MAX


def test_noalloc_rejects_more_rows_than_its_scratch():
    csr = rb.radial_mask_build(33, 3600, 128, sink=1)          # n = 118,800
    buf = torch.empty(64, dtype=torch.uint8, device="cuda")    # never dereferenced
    d = B.radial_desc()
    d.batch, d.heads, d.n_tokens, d.head_dim = 1, 40, 118800, 128   # 4,752,000 rows > 4,194,304
    d.stride_n, d.stride_h, d.stride_b = 128, 118800 * 128, 40 * 118800 * 128
    n0 = rb.radial_launch_count()
    ptr = ctypes.c_void_p(buf.data_ptr())
    st = B.load().radial_attn_bwd_noalloc(csr.handle, ctypes.byref(d), *([ptr] * 9), None)
    assert st == 2  # RADIAL_EUNSUPPORTED
    assert b"exceeds" in B.load().radial_last_error()
    assert rb.radial_launch_count() == n0
