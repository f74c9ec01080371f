"""The C ABI on the host: the shared library loads, exports every function
include/radial.h declares, and rejects invalid arguments before touching a
device.  No compute calls (runs without a GPU)."""

import ctypes
import os
import re

import pytest

import block_sparse_attention_csr_b200 as rb
from block_sparse_attention_csr_b200 import _binding as B
from block_sparse_attention_csr_b200 import build as build_mod

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build_mod.build()
    return B.load()


def _declared_functions():
    text = open(os.path.join(ROOT, "include", "radial.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"\b(radial_[a-z0-9_]+)\s*\(", text)
    return sorted(set(names))


def test_header_declares_expected_entry_points():
    names = _declared_functions()
    for n in ("radial_mask_build", "radial_attn_fwd", "radial_attn_bwd"):
        assert n in names
    assert set(names) == set(B.EXPORTED)


def test_library_exports_every_declared_symbol(lib):
    for n in _declared_functions():
        assert hasattr(lib, n), n


def test_symbols_are_c_linkage():
    out = os.popen(f"nm -D --defined-only {B.lib_path}").read()
    for n in _declared_functions():
        assert re.search(rf"\bT {n}$", out, flags=re.M), n


def test_params_default(lib):
    p = rb.radial_params_default()
    assert (p.sink, p.central_band, p.width_scale_num, p.width_scale_den, p.decay) == (1, 1, 2, 1, 0)
    assert list(p.reserved) == [0] * 3


def test_status_strings(lib):
    for s in range(6):
        assert lib.radial_status_str(s)


@pytest.mark.parametrize("args,status", [
    (dict(frames=0, tokens_per_frame=4, block=64), 1),
    (dict(frames=4, tokens_per_frame=0, block=64), 1),
    (dict(frames=4, tokens_per_frame=4, block=96), 2),
    (dict(frames=4, tokens_per_frame=4, block=128, central_band=-1), 1),
    (dict(frames=4, tokens_per_frame=4, block=128, width_scale=(2, 2)), 1),
    (dict(frames=4, tokens_per_frame=4, block=128, width_scale=(65, 1)), 1),
    (dict(frames=4, tokens_per_frame=4, block=128, decay=2), 1),
    (dict(frames=4, tokens_per_frame=4, block=128, sink=7), 1),
    (dict(frames=4, tokens_per_frame=4, block=128, reserved=[0, 0, 1]), 1),
    (dict(frames=1 << 16, tokens_per_frame=1 << 16, block=128), 1),
])
def test_mask_build_validation(lib, args, status):
    with pytest.raises(rb.RadialError) as e:
        rb.radial_mask_build(stream=0, **args)
    assert e.value.status == status


def test_null_arguments_are_rejected(lib):
    assert lib.radial_mask_build(4, 4, 64, None, None, None) == 1
    assert lib.radial_mask_build_dense(0, 64, ctypes.byref(ctypes.c_void_p()), None) == 1
    info = B.radial_csr_info_t()
    assert lib.radial_csr_info(None, ctypes.byref(info)) == 1
    d = B.radial_desc()
    assert lib.radial_attn_fwd(None, ctypes.byref(d), None, None, None, None, None, None) == 1
    assert lib.radial_attn_bwd(None, ctypes.byref(d), *([None] * 10), 0, None) == 1
    assert lib.radial_last_error()


def test_bwd_workspace_size(lib):
    d = B.radial_desc()
    d.batch, d.heads, d.n_tokens, d.head_dim = 1, 2, 1000, 128
    ws = lib.radial_attn_bwd_workspace_size(ctypes.byref(d))
    assert ws >= 2 * 1000 * 4          # one fp32 row sum per (head, token)
    assert ws % 256 == 0
    d.heads = 0
    assert lib.radial_attn_bwd_workspace_size(ctypes.byref(d)) == 0


def test_csr_free_null_is_noop(lib):
    lib.radial_csr_free(None)


def test_debug_build_exports_the_same_symbols(lib):
    """libradial_debug.so (-DRADIAL_DEBUG: device-side range checks of every
    index read from the mask's arrays) is the same ABI."""
    assert os.path.exists(build_mod.OUT_DEBUG)
    dbg = ctypes.CDLL(build_mod.OUT_DEBUG)
    for n in _declared_functions():
        assert hasattr(dbg, n), n
