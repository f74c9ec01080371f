"""The LoRA-adapted projection on the library's tensor-core GEMM
(radial_lora_fwd / radial_lora_bwd through the C ABI) against the fp64
reference oracle.lora (lora_linear, lora_linear_backward), on seeded bf16
inputs: y, dx, dA, dB, and u = s x A^T.

Shapes cover a token count with a row tail (not a multiple of the 128-row
tile), an output width with a column tail, ranks from 8 (below one 64-wide K
block) to 64, a strided x, and dx accumulated over two calls.

Tolerance, relative to each tensor's largest reference magnitude: max-abs
1e-2 and mean-abs 2e-3.  The operands are exact bf16 values and the GEMM
accumulates in fp32; what remains is the bf16 rounding of the stored outputs
and of the intermediates u = s x A^T and s dy B (2^-9 relative each).
"""

import numpy as np
import pytest
import torch

import block_sparse_attention_csr_b200 as rb
from oracle import lora as LO

pytestmark = pytest.mark.gpu
DEV = "cuda"
REL_MAX, REL_MEAN = 1e-2, 2e-3


def _cmp(got, ref, what):
    got = got.double().cpu().numpy()
    scale = max(1e-6, float(np.abs(ref).max()))
    err = np.abs(got - ref)
    assert np.isfinite(got).all(), what
    assert err.max() <= REL_MAX * scale, f"{what}: max-abs {err.max():.3e} vs scale {scale:.3e}"
    assert err.mean() <= REL_MEAN * scale, f"{what}: mean-abs {err.mean():.3e} vs scale {scale:.3e}"


def _draw(n, ci, co, r, seed, pad=0):
    g = torch.Generator(device="cpu").manual_seed(seed)
    xw = torch.randn(n, ci + pad, generator=g)
    t = {"x": xw[:, :ci] if pad else xw, "dy": torch.randn(n, co, generator=g),
         "W": torch.randn(co, ci, generator=g) / ci ** 0.5, "A": torch.randn(r, ci, generator=g) / ci ** 0.5,
         "B": torch.randn(co, r, generator=g) / r ** 0.5}
    dev = {k: v.to(torch.bfloat16).to(DEV) for k, v in t.items()}
    if pad:
        full = xw.to(torch.bfloat16).to(DEV)
        dev["x"] = full[:, :ci]            # strided rows: ld = ci + pad
    return dev


@pytest.mark.parametrize("n,ci,co,r,s,pad,seed", [
    (256, 128, 128, 8, 0.5, 0, 1),
    (600, 256, 256, 16, 1.0, 0, 2),
    (1000, 384, 200, 64, 0.25, 0, 3),     # row tail (1000 = 7 x 128 + 104), column tail (200)
    (513, 128, 256, 32, 2.0, 64, 4),      # odd token count, strided x
])
def test_projection_forward_and_backward(n, ci, co, r, s, pad, seed):
    t = _draw(n, ci, co, r, seed, pad)
    y, u = rb.radial_lora_fwd(t["x"], t["W"], t["A"], t["B"], s)
    dx, dA, dB = rb.radial_lora_bwd(t["dy"], t["x"], t["W"], t["A"], t["B"], u, s)
    rb.radial_device_status()
    x, dy, W, A, B = (t[k].double().cpu().numpy() for k in ("x", "dy", "W", "A", "B"))
    _cmp(u, s * (x @ A.T), "u")
    _cmp(y, LO.lora_linear(x, W, A, B, s), "y")
    rdx, rdA, rdB = LO.lora_linear_backward(x, W, A, B, s, dy)
    _cmp(dx, rdx, "dx")
    _cmp(dA, rdA, "dA")
    _cmp(dB, rdB, "dB")


def test_dx_accumulates():
    t = _draw(600, 256, 256, 16, 5)
    y, u = rb.radial_lora_fwd(t["x"], t["W"], t["A"], t["B"], 1.0)
    dx1, _, _ = rb.radial_lora_bwd(t["dy"], t["x"], t["W"], t["A"], t["B"], u, 1.0)
    dx2 = dx1.clone()
    rb.radial_lora_bwd(t["dy"], t["x"], t["W"], t["A"], t["B"], u, 1.0, dx=dx2, accumulate_dx=True)
    rb.radial_device_status()
    ref = 2.0 * dx1.double()
    assert (dx2.double() - ref).abs().max().item() <= 2.0 ** -7 * ref.abs().max().item()
