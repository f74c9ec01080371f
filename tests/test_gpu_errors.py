"""Error paths on a real device: invalid arguments are rejected on the host
with a status and launch nothing; a bounded device wait that runs out is
reported by radial_device_status and leaves the context usable."""

import pytest
import torch

import block_sparse_attention_csr_b200 as rb
from block_sparse_attention_csr_b200 import inputs as I

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module")
def setup():
    wl = I.small_workload("e", 1, 2, 128, 5, 200, 128, 41)
    q, k, v, do = I.draw(wl, device=DEV, backward=True)
    csr = rb.radial_mask_build(5, 200, 128, sink=1)
    return csr, q, k, v, do


def _status(fn):
    with pytest.raises(rb.RadialError) as e:
        fn()
    return e.value.status


def test_invalid_forward_arguments_launch_nothing(setup):
    csr, q, k, v, _ = setup
    n0 = rb.radial_launch_count()
    wrong_n = torch.empty(1, 2, 999, 128, dtype=torch.bfloat16, device=DEV)
    assert _status(lambda: rb.radial_attn_fwd(csr, wrong_n, wrong_n, wrong_n)) == 1
    odd_d = torch.empty(1, 2, 1000, 96, dtype=torch.bfloat16, device=DEV)
    assert _status(lambda: rb.radial_attn_fwd(csr, odd_d, odd_d, odd_d)) == 2
    # misaligned base pointer (offset by one element = 2 bytes)
    flat = torch.empty(1 * 2 * 1000 * 128 + 8, dtype=torch.bfloat16, device=DEV)
    mis = flat[1:1 + 2 * 1000 * 128].view(1, 2, 1000, 128)
    assert _status(lambda: rb.radial_attn_fwd(csr, mis, k, v)) == 1
    assert rb.radial_launch_count() == n0


def test_small_workspace_is_rejected(setup):
    csr, q, k, v, do = setup
    o, lse = rb.radial_attn_fwd(csr, q, k, v)
    need = rb.radial_attn_bwd_workspace_size(q)
    small = torch.empty(need - 256, dtype=torch.uint8, device=DEV)
    n0 = rb.radial_launch_count()
    assert _status(lambda: rb.radial_attn_bwd(csr, do, q, k, v, o, lse, workspace=small)) == 1
    assert rb.radial_launch_count() == n0


def test_bounded_wait_times_out_and_context_survives(setup):
    csr, q, k, v, _ = setup
    rb.radial_device_status()                      # clean slate
    rb.radial_selftest_bounded_wait(20)            # kernel gives up after 20 ms
    assert _status(lambda: rb.radial_device_status()) == 5
    rb.radial_device_status()                      # the flag was cleared
    o, lse = rb.radial_attn_fwd(csr, q, k, v)      # the context still works
    rb.radial_device_status()
    assert torch.isfinite(o.float()).all()


def test_backward_map_failure_launches_nothing(setup):
    """A batch stride of 2^40 elements passes the host checks (batch is 1, so
    it is never used to address memory) but exceeds what a TMA descriptor can
    encode.  The backward must report the failure before its first launch,
    leaving the workspace as it was."""
    import ctypes
    from block_sparse_attention_csr_b200 import _binding as B
    csr, q, k, v, do = setup
    o, lse = rb.radial_attn_fwd(csr, q, k, v)
    rb.radial_device_status()
    d = rb.make_desc(q)
    d.stride_b = 1 << 40
    dq, dk, dv = (torch.empty_like(x) for x in (q, k, v))
    ws = torch.full((rb.radial_attn_bwd_workspace_size(q),), 7, dtype=torch.uint8, device=DEV)
    n0 = rb.radial_launch_count()
    p = [ctypes.c_void_p(t.data_ptr()) for t in (do, q, k, v, o, lse, dq, dk, dv, ws)]
    st = B.load().radial_attn_bwd(csr.handle, ctypes.byref(d), *p, ctypes.c_size_t(ws.numel()),
                                  ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 4, B.load().radial_last_error()  # RADIAL_ECUDA from the descriptor encode
    assert rb.radial_launch_count() == n0
    torch.cuda.synchronize()
    assert bool((ws == 7).all())
