"""Seeded synthetic workloads and their input generators.

This module holds shapes, seeds and random draws only: none of the method's
arithmetic.  It is the one piece that both the CUDA path's callers (tests,
bench) and the CPU reference's callers use, so that both sides see the same
numbers.

Recipe (shared by every workload): one ``torch.Generator`` per workload,
seeded with the workload's seed; Q, K, V (and dO when a backward is run) are
drawn in that order as standard normal fp32 of shape ``[B, H, N, D]``,
multiplied by the workload's ``value_scale`` and rounded to bf16
(round-to-nearest-even, torch's ``.to(torch.bfloat16)``).  Small workloads draw
on the CPU; workloads whose fp32 draw would not fit comfortably in host memory
draw on the CUDA device with a CUDA generator (same recipe, different stream
of numbers), and a CPU reference then reads the rows it needs back from the
device tensors.

The shapes stand in for the latent token grids of the video models the pages
evaluate (Wan2.1-14B at 480p, HunyuanVideo at 720p and at 4x length); their
weights, prompts and activations are not used or reproduced.
"""

from __future__ import annotations

from dataclasses import dataclass, field

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    heads: int
    head_dim: int
    frames: int
    tokens_per_frame: int
    block: int
    seed: int
    value_scale: float = 1.0
    backward: bool = False
    grid: tuple = field(default=())  # spatial latent grid (rows, cols), informative

    @property
    def n(self) -> int:
        return self.frames * self.tokens_per_frame

    @property
    def shape(self):
        return (self.batch, self.heads, self.n, self.head_dim)


WORKLOADS = {
    # tiny CPU-checkable case (fp32 draws, consumed as bf16)
    "tiny": Workload("tiny", 1, 1, 64, 8, 64, 64, seed=0, backward=True, grid=(8, 8)),
    # Wan2.1-14B-shaped 480p self-attention: 21 latent frames of 30x52
    "wan480p": Workload("wan480p", 1, 40, 128, 21, 1560, 128, seed=1,
                        value_scale=2.0 ** -0.5, grid=(30, 52)),
    # HunyuanVideo-shaped 720p, 5 s: 33 latent frames of 45x80
    "hunyuan720p": Workload("hunyuan720p", 1, 24, 128, 33, 3600, 128, seed=2, grid=(45, 80)),
    # 4x-length HunyuanVideo-shaped LoRA fine-tuning step (forward + backward)
    "hunyuan720p_4x": Workload("hunyuan720p_4x", 1, 24, 128, 132, 3600, 128, seed=3,
                               backward=True, grid=(45, 80)),
}
for _f in (8, 16, 33, 66, 132):
    WORKLOADS[f"sweep_f{_f}"] = Workload(f"sweep_f{_f}", 1, 24, 128, _f, 3600, 128,
                                         seed=4 + _f, grid=(45, 80))


def small_workload(name, batch, heads, head_dim, frames, tokens_per_frame, block, seed,
                   value_scale=1.0, backward=True):
    """An ad-hoc workload for parity tests (same recipe as the named ones)."""
    return Workload(name, batch, heads, head_dim, frames, tokens_per_frame, block, seed,
                    value_scale, backward)


def draw(wl: Workload, device="cpu", backward=None):
    """Draw (q, k, v[, do]) as bf16 tensors [B, H, N, D] on ``device``.

    The generator lives on ``device`` ("cpu" or a CUDA device).
    """
    backward = wl.backward if backward is None else backward
    dev = torch.device(device)
    g = torch.Generator(device=dev)
    g.manual_seed(wl.seed)
    out = []
    for _ in range(4 if backward else 3):
        x = torch.randn(wl.shape, generator=g, device=dev, dtype=torch.float32)
        if wl.value_scale != 1.0:
            x.mul_(wl.value_scale)
        out.append(x.to(torch.bfloat16))
        del x
    return tuple(out)


def draw_fp32(wl: Workload, backward=None):
    """The fp32 draws themselves (CPU), before bf16 rounding (tiny cases)."""
    backward = wl.backward if backward is None else backward
    g = torch.Generator(device="cpu")
    g.manual_seed(wl.seed)
    out = []
    for _ in range(4 if backward else 3):
        x = torch.randn(wl.shape, generator=g, dtype=torch.float32)
        if wl.value_scale != 1.0:
            x.mul_(wl.value_scale)
        out.append(x)
    return tuple(out)


def draw_lora_layer(batch, heads, head_dim, frames, tokens_per_frame, rank, seed, device="cpu"):
    """Seeded synthetic inputs of one LoRA-adapted attention layer step, all
    bf16: activations x and upstream gradient dy [B, N, C] ~ N(0, 1); frozen
    projections W_p [C, C] ~ N(0, 1/C) (unit-variance outputs); adapters
    A_p [r, C] ~ N(0, 1/C) and B_p [C, r] ~ N(0, 1/r) for p in q, k, v, o.
    (Fine-tuning starts from B = 0; random B exercises the adapter path.)
    Drawn on the CPU in the order x, dy, then W, A, B per projection."""
    C = heads * head_dim
    N = frames * tokens_per_frame
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    out = {"x": torch.randn(batch, N, C, generator=g), "dy": torch.randn(batch, N, C, generator=g)}
    for p in ("q", "k", "v", "o"):
        out["W_" + p] = torch.randn(C, C, generator=g) / C ** 0.5
        out["A_" + p] = torch.randn(rank, C, generator=g) / C ** 0.5
        out["B_" + p] = torch.randn(C, rank, generator=g) / rank ** 0.5
    return {k: v.to(torch.bfloat16).to(device) for k, v in out.items()}
