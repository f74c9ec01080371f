"""Forward parity: the CUDA path (through the C ABI) against the fp64 CPU
reference on the same seeded bf16 inputs.

Tolerances (from the acceptance criteria of the workload definitions):
O max-abs <= 2e-2 and mean-abs <= 2e-3 against fp64; LSE max-abs <= 1e-3
(fp32 accumulation of at most 5e5 terms on logits of magnitude < 10: relative
error ~1e-6, so 1e-3 leaves three orders of margin while still catching a
wrong scale, base or mask).
"""

import os

import numpy as np
import pytest
import torch

import block_sparse_attention_csr_b200 as rb
from block_sparse_attention_csr_b200 import inputs as I
from oracle import attention as A
from tests import oracle_pool

pytestmark = pytest.mark.gpu

O_MAX, O_MEAN, LSE_MAX = 2e-2, 2e-3, 1e-3
DEV = "cuda"


def _run_gpu(q, k, v, f, s, block, sink, dense=False):
    csr = rb.radial_mask_build_dense(f * s, block) if dense else rb.radial_mask_build(f, s, block, sink=sink)
    o, lse = rb.radial_attn_fwd(csr, q, k, v)
    rb.radial_device_status()
    return o, lse


def _check(o_gpu, lse_gpu, o_ref, lse_ref, what):
    err = np.abs(o_gpu.astype(np.float64) - o_ref)
    lerr = np.abs(lse_gpu.astype(np.float64) - lse_ref)
    assert np.isfinite(o_gpu).all(), what
    assert err.max() <= O_MAX, f"{what}: O max-abs {err.max():.3e}"
    assert err.mean() <= O_MEAN, f"{what}: O mean-abs {err.mean():.3e}"
    assert lerr.max() <= LSE_MAX, f"{what}: LSE max-abs {lerr.max():.3e}"


def _full_check(q, k, v, f, s, block, sink, dense=False, what=""):
    o, lse = _run_gpu(q, k, v, f, s, block, sink, dense)
    ff, ss = (1, f * s) if dense else (f, s)
    o_ref, l_ref = A.radial_forward(q.float().cpu().numpy(), k.float().cpu().numpy(),
                                    v.float().cpu().numpy(), ff, ss, bool(sink) and not dense)
    _check(o.float().cpu().numpy(), lse.cpu().numpy(), o_ref, l_ref, what)


def test_tiny_config_all_rows():
    wl = I.WORKLOADS["tiny"]
    q32, k32, v32 = I.draw_fp32(wl, backward=False)
    q, k, v = (x.to(torch.bfloat16).to(DEV) for x in (q32, k32, v32))
    _full_check(q, k, v, wl.frames, wl.tokens_per_frame, wl.block, 1, what="tiny")


SMALL = [
    # batch, heads, head_dim, frames, tokens_per_frame, block, sink, seed
    (1, 2, 128, 5, 200, 128, 1, 11),     # ragged tail (1000 = 7*128 + 104)
    (2, 2, 64, 7, 300, 64, 0, 12),       # batch > 1, block 64, sink off
    (1, 1, 128, 32, 256, 64, 1, 13),     # many tiles, block 64 / d 128
    (1, 1, 64, 40, 3, 128, 1, 14),       # s < block: one tile spans many frames
    (1, 1, 128, 64, 4, 64, 0, 15),       # sampled-diagonal branch (width < 1)
    (1, 3, 128, 2, 700, 128, 0, 16),     # f <= 2: the mask is all-ones
    (1, 1, 64, 1, 1, 64, 1, 17),         # a single token
    (1, 2, 128, 9, 1000, 128, 1, 18),    # frames not aligned to tiles
    (1, 1, 128, 12, 1560, 128, 1, 19),   # Wan-like frame size, 12 frames
    (1, 1, 128, 24, 100, 128, 1, 20),    # 64 <= s < block: a tile spans up to three frames
    (1, 2, 64, 16, 64, 128, 0, 21),      # s = 64: 64-key halves aligned to frames
]


@pytest.mark.parametrize("Bn,H,D,f,s,block,sink,seed", SMALL)
def test_small_all_rows(Bn, H, D, f, s, block, sink, seed):
    wl = I.small_workload("t", Bn, H, D, f, s, block, seed)
    q, k, v = I.draw(wl, device=DEV, backward=False)
    _full_check(q, k, v, f, s, block, sink, what=f"{(Bn, H, D, f, s, block, sink)}")


def test_dense_mask_equals_dense_attention():
    wl = I.small_workload("d", 1, 2, 128, 1, 1500, 128, 21)
    q, k, v = I.draw(wl, device=DEV, backward=False)
    _full_check(q, k, v, 1, 1500, 128, 0, dense=True, what="dense")


def test_strided_layout():
    """[B, N, H, D] storage viewed as [B, H, N, D] (non-contiguous heads)."""
    g = torch.Generator(device="cpu").manual_seed(22)
    Bn, H, N, D, f, s = 1, 3, 1200, 128, 6, 200
    base = [torch.randn(Bn, N, H, D, generator=g).to(torch.bfloat16).to(DEV) for _ in range(3)]
    q, k, v = (t.permute(0, 2, 1, 3) for t in base)
    o = torch.empty(Bn, N, H, D, dtype=torch.bfloat16, device=DEV).permute(0, 2, 1, 3)
    csr = rb.radial_mask_build(f, s, 128, sink=1)
    o, lse = rb.radial_attn_fwd(csr, q, k, v, o=o)
    rb.radial_device_status()
    o_ref, l_ref = A.radial_forward(q.float().cpu().numpy(), k.float().cpu().numpy(),
                                    v.float().cpu().numpy(), f, s, True)
    _check(o.float().cpu().numpy(), lse.cpu().numpy(), o_ref, l_ref, "strided")


def test_repeated_calls_are_deterministic():
    wl = I.small_workload("r", 1, 4, 128, 9, 1000, 128, 23)
    q, k, v = I.draw(wl, device=DEV, backward=False)
    csr = rb.radial_mask_build(9, 1000, 128, sink=1)
    o1, l1 = rb.radial_attn_fwd(csr, q, k, v)
    o2, l2 = rb.radial_attn_fwd(csr, q, k, v)
    rb.radial_device_status()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def _sampled_check(name, rows_per_head, heads=None):
    wl = I.WORKLOADS[name]
    q, k, v = I.draw(wl, device=DEV, backward=False)
    csr = rb.radial_mask_build(wl.frames, wl.tokens_per_frame, wl.block, sink=1)
    o, lse = rb.radial_attn_fwd(csr, q, k, v)
    rb.radial_device_status()
    n = wl.n
    heads = range(wl.heads) if heads is None else heads
    tasks, keep = [], []
    scale = 1.0 / np.sqrt(wl.head_dim)
    for h in heads:
        rows = A.sample_runs(n, rows_per_head, wl.tokens_per_frame, wl.block, seed=1000 + h)
        ridx = torch.as_tensor(rows, device=DEV)
        tasks.append((q[0, h, ridx].float().cpu().numpy().astype(np.float64),
                      k[0, h].float().cpu().numpy(), v[0, h].float().cpu().numpy(),
                      rows, wl.frames, wl.tokens_per_frame, True, scale))
        keep.append((o[0, h, ridx].float().cpu().numpy(), lse[0, h, ridx].cpu().numpy()))
    res = oracle_pool.run("fwd_runs", tasks)
    o_g = np.concatenate([a for a, _ in keep])
    l_g = np.concatenate([b for _, b in keep])
    o_r = np.concatenate([a for a, _ in res])
    l_r = np.concatenate([b for _, b in res])
    _check(o_g, l_g, o_r, l_r, name)


def test_wan480p_sampled_rows():
    _sampled_check("wan480p", 4096)


def test_hunyuan720p_sampled_rows():
    _sampled_check("hunyuan720p", 4096)


@pytest.mark.slow
def test_hunyuan720p_4x_sampled_rows():
    _sampled_check("hunyuan720p_4x", int(os.environ.get("RADIAL_4X_ROWS", "4096")))


@pytest.mark.parametrize("frames", [8, 16, 66])
def test_sweep_sampled_rows(frames):
    """The scaling sweep's other frame counts (33 and 132 are the HunyuanVideo
    shapes above): 4096 sampled rows of every head."""
    _sampled_check(f"sweep_f{frames}", int(os.environ.get("RADIAL_SWEEP_ROWS", "4096")))


def test_many_work_items_all_rows():
    """8 heads x 36 query-tile pairs = 288 work items, about two per
    persistent CTA: every row of O and LSE against the reference."""
    wl = I.small_workload("fmany", 1, 8, 128, 9, 1000, 128, 24)
    q, k, v = I.draw(wl, device=DEV, backward=False)
    o, lse = _run_gpu(q, k, v, 9, 1000, 128, 1)
    rows = np.arange(wl.n)
    scale = 1.0 / np.sqrt(wl.head_dim)
    tasks = [(q[0, h].double().cpu().numpy(), k[0, h].float().cpu().numpy(), v[0, h].float().cpu().numpy(),
              rows, 9, 1000, True, scale) for h in range(8)]
    res = oracle_pool.run("fwd_rows", tasks)
    _check(o[0].float().cpu().numpy().reshape(-1, 128), lse[0].cpu().numpy().reshape(-1),
           np.concatenate([a for a, _ in res]), np.concatenate([b for _, b in res]), "many items")


@pytest.mark.parametrize("Bn,H,chunks,permuted", [(1, 5, 3, False), (2, 4, 4, False), (1, 6, 2, True), (1, 8, 6, False)])
def test_staged_forward_equals_device_forward(Bn, H, chunks, permuted):
    """radial_attn_fwd_staged (host buffers, copies overlapped with the
    attention group by group) gives bit for bit the device call's O and LSE:
    the same kernel runs on each group of heads.  `permuted` stores
    [B, N, H, D] viewed as [B, H, N, D], whose heads are not contiguous."""
    g = torch.Generator(device="cpu").manual_seed(31 + H)
    N, D, f, s = 1000, 128, 5, 200
    shape = (Bn, N, H, D) if permuted else (Bn, H, N, D)
    view = (lambda t: t.permute(0, 2, 1, 3)) if permuted else (lambda t: t)
    base = [torch.randn(shape, generator=g).to(torch.bfloat16) for _ in range(3)]
    host = [view(t.pin_memory()) for t in base]
    dev = [view(t.to(DEV)) for t in base]
    csr = rb.radial_mask_build(f, s, 128, sink=1)
    o_ref, l_ref = rb.radial_attn_fwd(csr, *dev)
    o_dev = view(torch.empty(shape, dtype=torch.bfloat16, device=DEV))
    o_host = view(torch.empty(shape, dtype=torch.bfloat16).pin_memory())
    o_h, l_h = rb.radial_attn_fwd_staged(csr, *host, *dev, o_host=o_host, o_dev=o_dev, chunks=chunks)
    torch.cuda.synchronize()
    rb.radial_device_status()
    assert torch.equal(o_h, o_ref.cpu()) and torch.equal(l_h, l_ref.cpu())
