"""Head sharding of one attention problem across ranks (one process per GPU).

Every (batch, head) unit of the masked attention (Eq.2 of the Radial
Attention review, jaehun.me §3) is independent of the others, and the radial
mask (§4.2) depends on token positions only, so one problem of H heads splits
across N ranks by heads with nothing exchanged on the data path: rank r runs
heads [r*H/N, (r+1)*H/N) on views of the same [B, H, N, D] tensors (dimension
1 is the head), and every rank builds the same mask.  This is how the
length-extension fine-tuning of §4.3 spreads one long sequence's attention
over several GPUs.

The one collective here, gather_heads, reassembles the full result on every
rank for callers that need it; it is not part of the attention itself.
"""

from __future__ import annotations


def head_range(heads: int, world: int, rank: int):
    """Heads [h0, h1) of `rank` in a balanced split of `heads` over `world`
    ranks (sizes differ by at most one; a rank may get none when
    world > heads)."""
    if world < 1 or not 0 <= rank < world or heads < 0:
        raise ValueError(f"bad split: heads={heads} world={world} rank={rank}")
    return rank * heads // world, (rank + 1) * heads // world


def shard(x, world: int, rank: int):
    """This rank's heads of a [B, H, ...] tensor, as a view (no copy).  The
    view keeps the parent's strides, which the library's descriptor takes as
    they are."""
    h0, h1 = head_range(x.shape[1], world, rank)
    return x[:, h0:h1]


def gather_heads(local, heads: int, world: int, group=None):
    """Concatenate every rank's head slice into the full [B, heads, ...]
    tensor on every rank (all_gather; NCCL for CUDA tensors, gloo for CPU).
    Slices of unequal size are padded to the largest for the exchange."""
    import torch
    import torch.distributed as dist

    sizes = [head_range(heads, world, r) for r in range(world)]
    width = max(h1 - h0 for h0, h1 in sizes)
    shape = list(local.shape)
    shape[1] = width
    buf = torch.zeros(shape, dtype=local.dtype, device=local.device)
    buf[:, :local.shape[1]] = local
    parts = [torch.empty_like(buf) for _ in range(world)]
    dist.all_gather(parts, buf.contiguous(), group=group)
    return torch.cat([p[:, :h1 - h0] for p, (h0, h1) in zip(parts, sizes)], dim=1)
