"""LoRA-adapted attention layer step (block_sparse_attention_csr_b200.lora):
projections on the library's tensor-core GEMM, radial attention in its
block-sparse kernels, all through the C ABI, against the fp64 layer
reference (oracle.lora) on the same seeded bf16 inputs.

The reference rounds to bf16 exactly where the device stores bf16 between
stages (q, k, v, the attention output, dO), so the remaining differences are
fp32-accumulated GEMMs, the bf16 low-rank intermediates and the attention
kernels' own error.  Tolerances,
relative to the largest reference magnitude of each tensor: max-abs 3e-2 and
mean-abs 3e-3 -- the attention's own bounds (2e-2 / 2e-3 on unit-scale O,
5e-2 on gradients) after one more bf16 GEMM stage (relative rounding 2^-9
per stored bf16 value, summed in fp32 over C or N terms).
"""

import numpy as np
import pytest
import torch

import block_sparse_attention_csr_b200 as rb
from block_sparse_attention_csr_b200 import inputs as I
from block_sparse_attention_csr_b200.lora import RadialLoRALayer
from oracle import lora as LO

pytestmark = pytest.mark.gpu
DEV = "cuda"
REL_MAX, REL_MEAN = 3e-2, 3e-3


def _bf16(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to(torch.bfloat16).to(torch.float64).numpy()


def _cmp(got, ref, what):
    got = got.float().cpu().numpy().astype(np.float64)
    scale = max(1e-6, float(np.abs(ref).max()))
    err = np.abs(got - ref)
    assert np.isfinite(got).all(), what
    assert err.max() <= REL_MAX * scale, f"{what}: max-abs {err.max():.3e} vs scale {scale:.3e}"
    assert err.mean() <= REL_MEAN * scale, f"{what}: mean-abs {err.mean():.3e} vs scale {scale:.3e}"


@pytest.mark.parametrize("heads,head_dim,frames,tps,block,rank,scale,seed", [
    (2, 64, 4, 64, 64, 8, 0.5, 7),
    (2, 128, 3, 200, 128, 16, 1.0, 8),   # ragged tail: 600 tokens, tiles of 128
])
def test_lora_layer_step(heads, head_dim, frames, tps, block, rank, scale, seed):
    t = I.draw_lora_layer(1, heads, head_dim, frames, tps, rank, seed, device=DEV)
    csr = rb.radial_mask_build(frames, tps, block, sink=1)
    layer = RadialLoRALayer(csr, heads, {k: v for k, v in t.items() if k.startswith("W_")},
                            {k: v for k, v in t.items() if k[:2] in ("A_", "B_")}, scale)
    y, ctx = layer.forward(t["x"])
    g = layer.backward(ctx, t["dy"])
    rb.radial_device_status()

    P = {k: v.double().cpu().numpy() for k, v in t.items() if k not in ("x", "dy")}
    P["s"] = scale
    x = t["x"].double().cpu().numpy()
    dy = t["dy"].double().cpu().numpy()
    y_ref, cache = LO.layer_forward(x, P, heads, frames, tps, True, rnd=_bf16)
    g_ref = LO.layer_backward(P, cache, dy, heads, frames, tps, True, rnd=_bf16)

    _cmp(y, y_ref, "y")
    _cmp(g["x"], g_ref["x"], "dx")
    for p in LO.PROJ:
        _cmp(g["A_" + p], g_ref["A_" + p], "dA_" + p)
        _cmp(g["B_" + p], g_ref["B_" + p], "dB_" + p)
