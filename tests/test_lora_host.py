"""Host-side checks of the LoRA layer (block_sparse_attention_csr_b200.lora)
and of its projection entry points: the head view of the projection outputs,
the ABI's argument validation (which rejects before any device work, so it
runs without a GPU) and the backward's workspace size.  The projections
themselves run on the library's tensor-core GEMM; their parity against the
fp64 reference is tests/test_gpu_gemm.py and tests/test_gpu_lora.py."""

import ctypes

import numpy as np
import torch

from block_sparse_attention_csr_b200 import _binding as B
from block_sparse_attention_csr_b200 import build as build_mod
from block_sparse_attention_csr_b200.lora import RadialLoRALayer
from oracle import lora as LO


def _layer(rng, C, r, s):
    W = {"W_" + p: torch.tensor(rng.standard_normal((C, C))) for p in LO.PROJ}
    AB = {}
    for p in LO.PROJ:
        AB["A_" + p] = torch.tensor(rng.standard_normal((r, C)))
        AB["B_" + p] = torch.tensor(rng.standard_normal((C, r)))
    return RadialLoRALayer(None, 4, W, AB, s), W, AB


def _lib():
    build_mod.build()
    return B.load()


def test_projection_arguments_are_validated_on_the_host():
    L = _lib()
    vp = ctypes.c_void_p
    nul = vp(0)
    # rank not a multiple of 8, bad sizes, null pointers: EINVAL before any device work
    assert L.radial_lora_fwd(100, 128, 128, 12, 1.0, nul, 128, nul, nul, nul, nul, 128, nul, None) == 1
    assert L.radial_lora_fwd(0, 128, 128, 16, 1.0, nul, 128, nul, nul, nul, nul, 128, nul, None) == 1
    assert L.radial_lora_fwd(100, 128, 128, 16, 1.0, nul, 128, nul, nul, nul, nul, 128, nul, None) == 1
    assert b"NULL" in L.radial_last_error()
    assert L.radial_lora_bwd(100, 128, 128, 16, 1.0, nul, 128, nul, 128, nul, nul, nul, nul, nul, 128, 2,
                             nul, nul, nul, ctypes.c_size_t(0), None) == 1


def test_backward_workspace_size():
    L = _lib()
    n, ci, co, r = 118800, 3072, 3072, 64
    got = L.radial_lora_bwd_workspace_size(n, ci, co, r)
    # transposed W, B, A, v, x, dy, u (bf16) and fp32 dA, dB accumulators
    need = 2 * (ci * co + r * co + ci * r + n * r + r * n + ci * n + co * n + r * n) + 4 * (r * ci + co * r)
    assert need <= got <= need + 10 * 256
    assert L.radial_lora_bwd_workspace_size(0, ci, co, r) == 0


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
