"""Host-side check of the LoRA layer's projection algebra
(block_sparse_attention_csr_b200.lora): the GEMM sequences of one adapted
projection and of its backward, run here on CPU float64 tensors, against the
fp64 layer reference.  (The attention between the projections needs the GPU
library; its parity is tests/test_gpu_lora.py.)"""

import numpy as np
import torch

from block_sparse_attention_csr_b200.lora import RadialLoRALayer
from oracle import lora as LO


def _layer(rng, C, r, s):
    W = {"W_" + p: torch.tensor(rng.standard_normal((C, C))) for p in LO.PROJ}
    AB = {}
    for p in LO.PROJ:
        AB["A_" + p] = torch.tensor(rng.standard_normal((r, C)))
        AB["B_" + p] = torch.tensor(rng.standard_normal((C, r)))
    return RadialLoRALayer(None, 4, W, AB, s), W, AB


def test_projection_and_backward_match_reference():
    rng = np.random.default_rng(3)
    C, r, n, s = 32, 4, 17, 0.375
    layer, W, AB = _layer(rng, C, r, s)
    x = torch.tensor(rng.standard_normal((n, C)))
    dy = torch.tensor(rng.standard_normal((n, C)))
    for p in LO.PROJ:
        Wp, Ap, Bp = W["W_" + p].numpy(), AB["A_" + p].numpy(), AB["B_" + p].numpy()
        np.testing.assert_allclose(layer._proj(x, p).numpy(), LO.lora_linear(x.numpy(), Wp, Ap, Bp, s),
                                   rtol=1e-12, atol=1e-12)
        dx, dA, dB = layer._proj_backward(x, p, dy)
        rdx, rdA, rdB = LO.lora_linear_backward(x.numpy(), Wp, Ap, Bp, s, dy.numpy())
        np.testing.assert_allclose(dx.numpy(), rdx, rtol=1e-12, atol=1e-11)
        np.testing.assert_allclose(dA.numpy(), rdA, rtol=1e-12, atol=1e-11)
        np.testing.assert_allclose(dB.numpy(), rdB, rtol=1e-12, atol=1e-11)


def test_head_view_is_the_channel_split():
    # [B*N, C] storage viewed as [B, H, N, D]: head h, token t, feature d is
    # channel h*D + d of token t
    layer, _, _ = _layer(np.random.default_rng(4), 32, 2, 1.0)
    t2 = torch.arange(2 * 5 * 32, dtype=torch.float64).view(2 * 5, 32)
    v = layer._heads_view(t2, 2, 5)
    assert tuple(v.shape) == (2, 4, 5, 8)
    for b, h, n, d in [(0, 0, 0, 0), (1, 3, 4, 7), (0, 2, 3, 5)]:
        assert v[b, h, n, d].item() == t2[b * 5 + n, h * 8 + d].item()
    assert v.stride(3) == 1
