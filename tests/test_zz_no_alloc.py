"""The backward's no-allocation entry point (radial_attn_bwd_noalloc).

It serves callers that cannot give the library a workspace: a plugin or
callback interface with no allocator, a process whose device memory is all
reserved by another framework's pool, or a latency-critical loop that must not
call cudaMalloc (it can synchronise the device).  Instead of a workspace it
uses a fixed device array inside the library.  It runs the same kernels in the
same order as the workspace entry point, radial_attn_bwd, and both are
deterministic, so its gradients must be bit-identical to that call's, on two
calls in a row (the second reuses the array the first one left behind).  A
call must also leave the device's free memory unchanged.  This file sorts last
so that a run stopping at its first failure has run every other test already.
"""

import ctypes

import pytest
import torch

import block_sparse_attention_csr_b200 as rb
from block_sparse_attention_csr_b200 import _binding as B
from block_sparse_attention_csr_b200 import inputs as I

pytestmark = pytest.mark.gpu


def _check_equal_twice(wl, f, s, block, sink):
    q, k, v, do = I.draw(wl, device="cuda", backward=True)
    csr = rb.radial_mask_build(f, s, block, sink=sink)
    o, lse = rb.radial_attn_fwd(csr, q, k, v)
    ref = rb.radial_attn_bwd(csr, do, q, k, v, o, lse)
    rb.radial_device_status()
    got = tuple(torch.empty_like(x) for x in (q, k, v))
    for call in range(2):
        for t in got:
            t.fill_(float("nan"))           # no stale output can pass
        torch.cuda.synchronize()
        free0, _ = torch.cuda.mem_get_info()
        rb.radial_attn_bwd_noalloc(csr, do, q, k, v, o, lse, *got)
        rb.radial_device_status()
        free1, _ = torch.cuda.mem_get_info()
        for name, r, g in zip(("dQ", "dK", "dV"), ref, got):
            assert torch.equal(r, g), f"call {call}: {name} differs from radial_attn_bwd"
        if call == 1:
            # the first call may load the module and look up the array; after
            # it, a call allocates nothing
            assert free1 == free0, f"free device memory changed by {free0 - free1} bytes"


def test_noalloc_backward_equals_workspace_backward_twice():
    wl = I.small_workload("noalloc", 1, 2, 128, 9, 1000, 128, 51)
    _check_equal_twice(wl, 9, 1000, 128, 1)


def test_noalloc_backward_d64_block64():
    wl = I.small_workload("noalloc64", 2, 2, 64, 7, 300, 64, 52)
    _check_equal_twice(wl, 7, 300, 64, 0)


def test_noalloc_rejects_more_rows_than_its_scratch():
    csr = rb.radial_mask_build(5, 200, 128, sink=1)             # n = 1000
    buf = torch.empty(64, dtype=torch.uint8, device="cuda")    # never dereferenced
    d = B.radial_desc()
    d.batch, d.heads, d.n_tokens, d.head_dim = 1, 4200, 1000, 128   # 4,200,000 rows > 4,194,304
    d.stride_n, d.stride_h, d.stride_b = 128, 1000 * 128, 4200 * 1000 * 128
    n0 = rb.radial_launch_count()
    ptr = ctypes.c_void_p(buf.data_ptr())
    st = B.load().radial_attn_bwd_noalloc(csr.handle, ctypes.byref(d), *([ptr] * 9), None)
    assert st == 2  # RADIAL_EUNSUPPORTED
    assert b"exceeds" in B.load().radial_last_error()
    assert rb.radial_launch_count() == n0
