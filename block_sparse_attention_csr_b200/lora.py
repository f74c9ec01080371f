"""One LoRA-adapted attention layer step of a video DiT on B200.

The Radial Attention review (§4.3) extends a pretrained video diffusion model
to longer videos by fine-tuning LoRA adapters on the Q/K/V/O projections of
its attention layers while the attention itself runs under the radial mask.
This module is that layer step: per projection p in q, k, v, o

    y = x W_p^T + s (x A_p^T) B_p^T          (W_p frozen, A_p / B_p trained)

around the block-sparse radial attention, forward and backward (dx and the
adapter gradients dA_p, dB_p; W_p gets none).

Everything runs in libradial through the C ABI: the projections on its
tensor-core GEMM (radial_lora_fwd / radial_lora_bwd: bf16 operands, fp32
accumulation, the low-rank update fused into the same accumulator), the
attention forward and backward in its block-sparse kernels.  Heads are split
from the channel axis as [B, N, H, D]; the attention sees strided
[B, H, N, D] views of the projection outputs, so no tensor is copied or
transposed between the projections and the attention.
"""

from __future__ import annotations

from . import _binding as _b

PROJ = ("q", "k", "v", "o")


class RadialLoRALayer:
    """LoRA on Q/K/V/O around radial attention.

    ``weights``: W_q, W_k, W_v, W_o, each [C, C] bf16 (frozen, out x in).
    ``adapters``: A_p [r, C] and B_p [C, r] bf16 for p in q, k, v, o.
    ``scale``: the adapter scale s (alpha / r).  ``csr`` is the radial mask of
    the layer's token grid (``radial_mask_build``); C = heads * head_dim.
    """

    def __init__(self, csr, heads, weights, adapters, scale):
        self.csr = csr
        self.heads = int(heads)
        self.W = {p: weights["W_" + p] for p in PROJ}
        self.A = {p: adapters["A_" + p] for p in PROJ}
        self.B = {p: adapters["B_" + p] for p in PROJ}
        self.s = float(scale)
        C = self.W["q"].shape[0]
        if C % self.heads:
            raise ValueError("hidden size must be a multiple of heads")
        self.head_dim = C // self.heads
        self._ws = None  # backward workspace, kept across steps

    def _proj(self, x2, p, y=None):
        """(y, u): the projection and its saved low-rank activation u = s x A^T."""
        return _b.radial_lora_fwd(x2, self.W[p], self.A[p], self.B[p], self.s, y=y)

    def _proj_backward(self, x2, p, dy2, u, dx=None, accumulate=False):
        import torch
        n, C = x2.shape
        need = int(_b.load().radial_lora_bwd_workspace_size(n, C, self.W[p].shape[0], self.A[p].shape[0]))
        if self._ws is None or self._ws.numel() < need:
            self._ws = torch.empty(need, dtype=torch.uint8, device=x2.device)
        return _b.radial_lora_bwd(dy2, x2, self.W[p], self.A[p], self.B[p], u, self.s, dx=dx,
                                  accumulate_dx=accumulate, workspace=self._ws)

    def _heads_view(self, t2, Bn, N):
        return t2.view(Bn, N, self.heads, self.head_dim).permute(0, 2, 1, 3)

    def forward(self, x):
        """x [B, N, C] bf16 -> (y [B, N, C] bf16, ctx for backward)."""
        import torch
        Bn, N, C = x.shape
        x2 = x.reshape(Bn * N, C)
        u = {}
        heads = {}
        for p in ("q", "k", "v"):
            y2, u[p] = self._proj(x2, p)
            heads[p] = self._heads_view(y2, Bn, N)
        o2 = torch.empty(Bn * N, C, dtype=torch.bfloat16, device=x.device)
        o = self._heads_view(o2, Bn, N)
        lse = torch.empty(Bn, self.heads, N, dtype=torch.float32, device=x.device)
        _b.radial_attn_fwd(self.csr, heads["q"], heads["k"], heads["v"], o=o, lse=lse)
        y2, u["o"] = self._proj(o2, "o")
        return y2.view(Bn, N, C), (x2, heads["q"], heads["k"], heads["v"], o, o2, lse, u, Bn, N)

    def backward(self, ctx, dy):
        """Upstream dy [B, N, C] -> dict with "x" [B, N, C] and A_p, B_p grads."""
        import torch
        x2, q, k, v, o, o2, lse, u, Bn, N = ctx
        C = x2.shape[1]
        grads = {}
        da2, grads["A_o"], grads["B_o"] = self._proj_backward(o2, "o", dy.reshape(Bn * N, C), u["o"])
        do = self._heads_view(da2, Bn, N)
        d2 = {p: torch.empty(Bn * N, C, dtype=torch.bfloat16, device=dy.device) for p in ("q", "k", "v")}
        _b.radial_attn_bwd(self.csr, do, q, k, v, o, lse, dq=self._heads_view(d2["q"], Bn, N),
                           dk=self._heads_view(d2["k"], Bn, N), dv=self._heads_view(d2["v"], Bn, N))
        dx = torch.empty(Bn * N, C, dtype=torch.bfloat16, device=dy.device)
        for i, p in enumerate(("q", "k", "v")):
            _, grads["A_" + p], grads["B_" + p] = self._proj_backward(x2, p, d2[p], u[p], dx=dx, accumulate=i > 0)
        grads["x"] = dx.view(Bn, N, C)
        return grads
