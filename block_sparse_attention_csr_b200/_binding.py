"""ctypes binding of libradial: argument marshalling only.

Every step of the attention path runs in the library's CUDA kernels; this
module turns torch tensors into pointers, strides and the CUDA stream handle,
calls the C ABI (include/radial.h) by the same names, and raises on a non-OK
status.  It never computes anything itself and has no fallback: if the
shared library is missing it raises.
"""

from __future__ import annotations

import ctypes
import os
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_NAME = "libradial.so"
# RADIAL_LIBRARY names another build of the same library (for instance the
# bounds-checking libradial_debug.so); by default the in-tree release build.
lib_path = os.environ.get("RADIAL_LIBRARY") or os.path.join(_HERE, LIB_NAME)

RADIAL_OK = 0
STATUS_NAMES = {0: "RADIAL_OK", 1: "RADIAL_EINVAL", 2: "RADIAL_EUNSUPPORTED", 3: "RADIAL_ENOMEM",
                4: "RADIAL_ECUDA", 5: "RADIAL_EDEVICE"}

EXPORTED = (
    "radial_params_default", "radial_mask_build", "radial_mask_build_dense", "radial_csr_info",
    "radial_csr_copy_to_host", "radial_csr_free", "radial_attn_fwd",
    "radial_attn_bwd_workspace_size", "radial_attn_bwd", "radial_device_status",
    "radial_status_str", "radial_last_error", "radial_launch_count", "radial_selftest_bounded_wait",
    "radial_attn_bwd_noalloc", "radial_attn_fwd_staged", "radial_lora_fwd", "radial_lora_bwd_workspace_size", "radial_lora_bwd",
)


class RadialError(RuntimeError):
    def __init__(self, status, where, msg):
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}: {msg}")
        self.status = status


class radial_params(ctypes.Structure):
    _fields_ = [("sink", ctypes.c_int32), ("central_band", ctypes.c_int32),
                ("width_scale_num", ctypes.c_int32), ("width_scale_den", ctypes.c_int32),
                ("decay", ctypes.c_int32), ("reserved", ctypes.c_int32 * 3)]


class radial_csr_info_t(ctypes.Structure):
    _fields_ = [("frames", ctypes.c_int32), ("tokens_per_frame", ctypes.c_int32),
                ("n_tokens", ctypes.c_int32), ("block", ctypes.c_int32),
                ("n_blocks", ctypes.c_int32), ("sink", ctypes.c_int32), ("dense", ctypes.c_int32),
                ("reserved", ctypes.c_int32), ("nnz", ctypes.c_int64), ("n_full", ctypes.c_int64),
                ("allowed_pairs", ctypes.c_int64)]


class radial_desc(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("heads", ctypes.c_int32), ("n_tokens", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("stride_b", ctypes.c_int64),
                ("stride_h", ctypes.c_int64), ("stride_n", ctypes.c_int64),
                ("scale", ctypes.c_float), ("reserved", ctypes.c_int32)]


_lib = None
_lock = threading.Lock()


def load(path=None):
    """Load the shared library (once).  Raises if it is absent."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        p = path or lib_path
        if not os.path.exists(p):
            raise RuntimeError(f"{os.path.basename(p)} not built at {p}; run block_sparse_attention_csr_b200.build")
        L = ctypes.CDLL(p)
        vp, i32, i64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
        L.radial_params_default.argtypes = [ctypes.POINTER(radial_params)]
        L.radial_params_default.restype = None
        L.radial_mask_build.argtypes = [i32, i32, i32, ctypes.POINTER(radial_params),
                                        ctypes.POINTER(vp), vp]
        L.radial_mask_build.restype = ctypes.c_int
        L.radial_mask_build_dense.argtypes = [i32, i32, ctypes.POINTER(vp), vp]
        L.radial_mask_build_dense.restype = ctypes.c_int
        L.radial_csr_info.argtypes = [vp, ctypes.POINTER(radial_csr_info_t)]
        L.radial_csr_info.restype = ctypes.c_int
        L.radial_csr_copy_to_host.argtypes = [vp] * 9
        L.radial_csr_copy_to_host.restype = ctypes.c_int
        L.radial_csr_free.argtypes = [vp]
        L.radial_csr_free.restype = None
        L.radial_attn_fwd.argtypes = [vp, ctypes.POINTER(radial_desc)] + [vp] * 6
        L.radial_attn_fwd.restype = ctypes.c_int
        L.radial_attn_fwd_staged.argtypes = [vp, ctypes.POINTER(radial_desc)] + [vp] * 10 + [i32, vp]
        L.radial_attn_fwd_staged.restype = ctypes.c_int
        L.radial_attn_bwd_workspace_size.argtypes = [ctypes.POINTER(radial_desc)]
        L.radial_attn_bwd_workspace_size.restype = sz
        L.radial_attn_bwd.argtypes = [vp, ctypes.POINTER(radial_desc)] + [vp] * 10 + [sz, vp]
        L.radial_attn_bwd.restype = ctypes.c_int
        L.radial_attn_bwd_noalloc.argtypes = [vp, ctypes.POINTER(radial_desc)] + [vp] * 10
        L.radial_attn_bwd_noalloc.restype = ctypes.c_int
        L.radial_lora_fwd.argtypes = [i64, i32, i32, i32, ctypes.c_float, vp, i64, vp, vp, vp, vp, i64, vp, vp]
        L.radial_lora_fwd.restype = ctypes.c_int
        L.radial_lora_bwd_workspace_size.argtypes = [i64, i32, i32, i32]
        L.radial_lora_bwd_workspace_size.restype = sz
        L.radial_lora_bwd.argtypes = [i64, i32, i32, i32, ctypes.c_float, vp, i64, vp, i64, vp, vp, vp, vp, vp, i64,
                                      i32, vp, vp, vp, sz, vp]
        L.radial_lora_bwd.restype = ctypes.c_int
        L.radial_device_status.argtypes = [vp]
        L.radial_device_status.restype = ctypes.c_int
        L.radial_status_str.argtypes = [ctypes.c_int]
        L.radial_status_str.restype = ctypes.c_char_p
        L.radial_last_error.argtypes = []
        L.radial_last_error.restype = ctypes.c_char_p
        L.radial_selftest_bounded_wait.argtypes = [ctypes.c_uint32, vp]
        L.radial_selftest_bounded_wait.restype = ctypes.c_int
        L.radial_launch_count.argtypes = []
        L.radial_launch_count.restype = i64
        _lib = L
        return L


def _check(status, where):
    if status != RADIAL_OK:
        raise RadialError(status, where, load().radial_last_error().decode())


def _stream(stream):
    if stream is None:
        import torch
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return ctypes.c_void_p(stream)
    return ctypes.c_void_p(stream.cuda_stream)


def _ptr(t):
    return ctypes.c_void_p(0 if t is None else t.data_ptr())


class Csr:
    """Owner of a device-side radial_csr handle."""

    def __init__(self, handle):
        self._h = handle

    @property
    def handle(self):
        return self._h

    def info(self):
        return radial_csr_info(self)

    def __del__(self):
        try:
            if self._h is not None and _lib is not None:
                _lib.radial_csr_free(self._h)
        except Exception:
            pass
        self._h = None


def radial_params_default():
    p = radial_params()
    load().radial_params_default(ctypes.byref(p))
    return p


DECAYS = {"radial": 0, "harmonic": 1}


def radial_mask_build(frames, tokens_per_frame, block, sink=1, central_band=1, width_scale=(2, 1),
                      decay="radial", stream=None, reserved=None):
    """width_scale: (num, den) of the band-to-band width ratio; decay: "radial" or "harmonic"."""
    p = radial_params_default()
    num, den = (width_scale, 1) if isinstance(width_scale, int) else width_scale
    p.sink, p.central_band = int(sink), int(central_band)
    p.width_scale_num, p.width_scale_den = int(num), int(den)
    p.decay = DECAYS[decay] if isinstance(decay, str) else int(decay)
    if reserved is not None:
        for i, r in enumerate(reserved):
            p.reserved[i] = int(r)
    h = ctypes.c_void_p()
    _check(load().radial_mask_build(int(frames), int(tokens_per_frame), int(block), ctypes.byref(p),
                                    ctypes.byref(h), _stream(stream)), "radial_mask_build")
    return Csr(h)


def radial_mask_build_dense(n_tokens, block, stream=None):
    h = ctypes.c_void_p()
    _check(load().radial_mask_build_dense(int(n_tokens), int(block), ctypes.byref(h), _stream(stream)),
           "radial_mask_build_dense")
    return Csr(h)


def radial_csr_info(csr):
    info = radial_csr_info_t()
    _check(load().radial_csr_info(csr.handle, ctypes.byref(info)), "radial_csr_info")
    return {f: getattr(info, f) for f, _ in radial_csr_info_t._fields_}


def radial_csr_copy_to_host(csr):
    """All mask arrays as numpy (user block size)."""
    info = radial_csr_info(csr)
    nb, nnz = info["n_blocks"], info["nnz"]
    out = dict(
        row_ptr=np.empty(nb + 1, np.int32), col_idx=np.empty(nnz, np.int32), kind=np.empty(nnz, np.uint8),
        col_ptr=np.empty(nb + 1, np.int32), row_idx=np.empty(nnz, np.int32), kind_t=np.empty(nnz, np.uint8),
        row_order=np.empty(nb, np.int32), col_order=np.empty(nb, np.int32))
    a = [ctypes.c_void_p(out[k].ctypes.data) for k in
         ("row_ptr", "col_idx", "kind", "col_ptr", "row_idx", "kind_t", "row_order", "col_order")]
    _check(load().radial_csr_copy_to_host(csr.handle, *a), "radial_csr_copy_to_host")
    return out


def make_desc(q, scale=None):
    """radial_desc of a [B, H, N, D] bf16 tensor (D contiguous)."""
    if q.dim() != 4:
        raise ValueError("expected a [batch, heads, n_tokens, head_dim] tensor")
    if q.stride(3) != 1:
        raise ValueError("head_dim must be contiguous")
    d = radial_desc()
    d.batch, d.heads, d.n_tokens, d.head_dim = (int(x) for x in q.shape)
    d.stride_b, d.stride_h, d.stride_n = q.stride(0), q.stride(1), q.stride(2)
    d.scale = 0.0 if scale is None else float(scale)
    d.reserved = 0
    return d


def _same_layout(ref, *ts):
    import torch
    for t in ts:
        if t is None:
            continue
        if t.shape != ref.shape or t.stride() != ref.stride() or t.dtype != torch.bfloat16 or not t.is_cuda:
            raise ValueError("all attention tensors must be CUDA bf16 with identical shape and strides")


def radial_attn_fwd(csr, q, k, v, o=None, lse=None, scale=None, stream=None):
    """Forward through the C ABI.  Allocates o / lse (torch) when not given."""
    import torch
    if o is None:
        o = torch.empty_like(q)
    if lse is None:
        lse = torch.empty(q.shape[:3], dtype=torch.float32, device=q.device)
    _same_layout(q, k, v, o)
    desc = make_desc(q, scale)
    _check(load().radial_attn_fwd(csr.handle, ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(o),
                                  _ptr(lse), _stream(stream)), "radial_attn_fwd")
    return o, lse


def radial_attn_fwd_staged(csr, q_host, k_host, v_host, q_dev, k_dev, v_dev, o_host=None, lse_host=None,
                           o_dev=None, lse_dev=None, chunks=4, scale=None, stream=None):
    """Forward of host (pinned) tensors with the copies overlapped with the
    attention, group of heads by group of heads.  Host and device tensors
    share one [B, H, N, D] layout; the outputs land in o_host / lse_host
    (allocated pinned when not given).  Returns (o_host, lse_host)."""
    import torch
    if o_host is None:
        o_host = torch.empty_strided(q_host.shape, q_host.stride(), dtype=torch.bfloat16).pin_memory()
    if lse_host is None:
        lse_host = torch.empty(q_host.shape[:3], dtype=torch.float32).pin_memory()
    if o_dev is None:
        o_dev = torch.empty_like(q_dev)
    if lse_dev is None:
        lse_dev = torch.empty(q_dev.shape[:3], dtype=torch.float32, device=q_dev.device)
    _same_layout(q_dev, k_dev, v_dev, o_dev)
    for t in (q_host, k_host, v_host, o_host):
        if t.shape != q_dev.shape or t.stride() != q_dev.stride() or t.dtype != torch.bfloat16 or t.is_cuda:
            raise ValueError("host tensors must be CPU bf16 with the device tensors' shape and strides")
    desc = make_desc(q_dev, scale)
    _check(load().radial_attn_fwd_staged(csr.handle, ctypes.byref(desc), _ptr(q_host), _ptr(k_host), _ptr(v_host),
                                         _ptr(o_host), _ptr(lse_host), _ptr(q_dev), _ptr(k_dev), _ptr(v_dev),
                                         _ptr(o_dev), _ptr(lse_dev), int(chunks), _stream(stream)),
           "radial_attn_fwd_staged")
    return o_host, lse_host


def radial_attn_bwd_workspace_size(q):
    desc = make_desc(q)
    return int(load().radial_attn_bwd_workspace_size(ctypes.byref(desc)))


def radial_attn_bwd(csr, do, q, k, v, o, lse, dq=None, dk=None, dv=None, workspace=None, scale=None,
                    stream=None):
    """Backward through the C ABI.  Allocates outputs / workspace (torch) when not given."""
    import torch
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    _same_layout(q, k, v, o, do, dq, dk, dv)
    desc = make_desc(q, scale)
    need = int(load().radial_attn_bwd_workspace_size(ctypes.byref(desc)))
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    _check(load().radial_attn_bwd(csr.handle, ctypes.byref(desc), _ptr(do), _ptr(q), _ptr(k), _ptr(v),
                                  _ptr(o), _ptr(lse), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(workspace),
                                  ctypes.c_size_t(workspace.numel() * workspace.element_size()),
                                  _stream(stream)), "radial_attn_bwd")
    return dq, dk, dv


def radial_attn_bwd_noalloc(csr, do, q, k, v, o, lse, dq=None, dk=None, dv=None, scale=None, stream=None):
    """Backward through the no-allocation entry point (no workspace; the library
    uses its fixed device scratch).  Allocates the outputs (torch) when not given."""
    import torch
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    _same_layout(q, k, v, o, do, dq, dk, dv)
    desc = make_desc(q, scale)
    _check(load().radial_attn_bwd_noalloc(csr.handle, ctypes.byref(desc), _ptr(do), _ptr(q), _ptr(k), _ptr(v),
                                          _ptr(o), _ptr(lse), _ptr(dq), _ptr(dk), _ptr(dv), _stream(stream)),
           "radial_attn_bwd_noalloc")
    return dq, dk, dv


def _rows(t, what):
    """(rows, cols, row stride) of a 2-D bf16 CUDA tensor with unit column stride."""
    import torch
    if t.dim() != 2 or t.stride(1) != 1 or t.dtype != torch.bfloat16 or not t.is_cuda:
        raise ValueError(f"{what}: expected a 2-D CUDA bf16 tensor with contiguous rows")
    return t.shape[0], t.shape[1], t.stride(0)


def radial_lora_fwd(x, W, A, B, scale, y=None, u=None, stream=None):
    """y = x W^T + s (x A^T) B^T on the library's tensor-core GEMMs.
    x [n, c_in], W [c_out, c_in], A [r, c_in], B [c_out, r].  Returns (y, u)
    with u = s x A^T, which radial_lora_bwd takes back."""
    import torch
    n, c_in, ldx = _rows(x, "x")
    c_out, r = W.shape[0], A.shape[0]
    for t, shape, nm in ((W, (c_out, c_in), "W"), (A, (r, c_in), "A"), (B, (c_out, r), "B")):
        if tuple(t.shape) != shape or not t.is_contiguous():
            raise ValueError(f"{nm}: expected a contiguous {shape} tensor")
    y = torch.empty(n, c_out, dtype=torch.bfloat16, device=x.device) if y is None else y
    u = torch.empty(n, r, dtype=torch.bfloat16, device=x.device) if u is None else u
    _, _, ldy = _rows(y, "y")
    _check(load().radial_lora_fwd(n, c_in, c_out, r, float(scale), _ptr(x), ldx, _ptr(W), _ptr(A), _ptr(B),
                                  _ptr(y), ldy, _ptr(u), _stream(stream)), "radial_lora_fwd")
    return y, u


def radial_lora_bwd(dy, x, W, A, B, u, scale, dx=None, accumulate_dx=False, dA=None, dB=None, workspace=None,
                    stream=None):
    """(dx, dA, dB) of radial_lora_fwd for upstream dy [n, c_out]; with
    accumulate_dx the result is added to the given dx."""
    import torch
    n, c_out, lddy = _rows(dy, "dy")
    _, c_in, ldx = _rows(x, "x")
    r = A.shape[0]
    dx = torch.empty(n, c_in, dtype=torch.bfloat16, device=x.device) if dx is None else dx
    dA = torch.empty(r, c_in, dtype=torch.bfloat16, device=x.device) if dA is None else dA
    dB = torch.empty(c_out, r, dtype=torch.bfloat16, device=x.device) if dB is None else dB
    _, _, lddx = _rows(dx, "dx")
    need = int(load().radial_lora_bwd_workspace_size(n, c_in, c_out, r))
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=x.device)
    _check(load().radial_lora_bwd(n, c_in, c_out, r, float(scale), _ptr(dy), lddy, _ptr(x), ldx, _ptr(W), _ptr(A),
                                  _ptr(B), _ptr(u), _ptr(dx), lddx, 1 if accumulate_dx else 0, _ptr(dA), _ptr(dB),
                                  _ptr(workspace), ctypes.c_size_t(workspace.numel() * workspace.element_size()),
                                  _stream(stream)), "radial_lora_bwd")
    return dx, dA, dB


def radial_device_status(stream=None):
    _check(load().radial_device_status(_stream(stream)), "radial_device_status")


def radial_selftest_bounded_wait(limit_ms=20, stream=None):
    _check(load().radial_selftest_bounded_wait(int(limit_ms), _stream(stream)), "radial_selftest_bounded_wait")


def radial_launch_count():
    return int(load().radial_launch_count())
