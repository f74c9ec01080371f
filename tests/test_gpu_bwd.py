"""Backward parity: dQ, dK, dV from the CUDA path (C ABI) against the fp64 CPU
reference computed from the same bf16 inputs (the reference recomputes its
own O and LSE; nothing it uses comes from the device path).

Tolerance: max-abs 5e-2 on every gradient (the acceptance criterion of the
workload definitions).  At the 4x-length shape, where the reference cannot
afford every key's column, dQ is checked on sampled rows and dK / dV through
identities that hold at any size: sum over keys of dK is 0 (each row of dS
sums to zero) and sum over keys of dV equals sum over queries of dO (each row
of P sums to one).
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

G_MAX = 5e-2
DEV = "cuda"


def _gpu_fwd_bwd(q, k, v, do, csr):
    o, lse = rb.radial_attn_fwd(csr, q, k, v)
    dq, dk, dv = rb.radial_attn_bwd(csr, do, q, k, v, o, lse)
    rb.radial_device_status()
    return o, lse, dq, dk, dv


def _full(q, k, v, do, f, s, block, sink, what, dense=False):
    csr = rb.radial_mask_build_dense(f * s, block) if dense else rb.radial_mask_build(f, s, block, sink=sink)
    _, _, dq, dk, dv = _gpu_fwd_bwd(q, k, v, do, csr)
    x = [t.float().cpu().numpy() for t in (q, k, v, do)]
    ff, ss = (1, f * s) if dense else (f, s)
    sk = bool(sink) and not dense
    o_ref, l_ref = A.radial_forward(x[0], x[1], x[2], ff, ss, sk)
    g_ref = A.radial_backward(x[0], x[1], x[2], o_ref, x[3], l_ref, ff, ss, sk)
    for name, g, r in zip(("dQ", "dK", "dV"), (dq, dk, dv), g_ref):
        gg = g.float().cpu().numpy()
        assert np.isfinite(gg).all(), f"{what} {name}"
        err = np.abs(gg - r).max()
        assert err <= G_MAX, f"{what}: {name} max-abs {err:.3e}"


def test_tiny_config_all_gradients():
    wl = I.WORKLOADS["tiny"]
    q, k, v, do = (x.to(torch.bfloat16).to(DEV) for x in I.draw_fp32(wl, backward=True))
    _full(q, k, v, do, wl.frames, wl.tokens_per_frame, wl.block, 1, "tiny")


SMALL = [
    (1, 2, 128, 5, 200, 128, 1, 31),
    (2, 2, 64, 7, 300, 64, 0, 32),
    (1, 1, 128, 32, 256, 64, 1, 33),
    (1, 1, 64, 40, 3, 128, 1, 34),
    (1, 1, 128, 64, 4, 64, 0, 35),
    (1, 2, 128, 2, 700, 128, 0, 36),
    (1, 1, 64, 1, 1, 64, 1, 37),
    (1, 2, 128, 9, 1000, 128, 1, 38),
    (1, 1, 128, 24, 100, 128, 1, 39),   # 64 <= s < block: a tile spans up to three frames
    (1, 2, 64, 16, 64, 128, 0, 40),     # s = 64: 64-token halves aligned to frames
]


@pytest.mark.parametrize("Bn,H,D,f,s,block,sink,seed", SMALL)
def test_small_all_gradients(Bn, H, D, f, s, block, sink, seed):
    wl = I.small_workload("b", Bn, H, D, f, s, block, seed)
    q, k, v, do = I.draw(wl, device=DEV, backward=True)
    _full(q, k, v, do, f, s, block, sink, f"{(Bn, H, D, f, s, block, sink)}")


def test_dense_mask_gradients():
    wl = I.small_workload("bd", 1, 1, 128, 1, 1100, 128, 39)
    q, k, v, do = I.draw(wl, device=DEV, backward=True)
    _full(q, k, v, do, 1, 1100, 128, 0, "dense", dense=True)


def test_backward_is_deterministic():
    wl = I.small_workload("bdet", 1, 2, 128, 9, 1000, 128, 40)
    q, k, v, do = I.draw(wl, device=DEV, backward=True)
    csr = rb.radial_mask_build(9, 1000, 128, sink=1)
    a = _gpu_fwd_bwd(q, k, v, do, csr)
    b = _gpu_fwd_bwd(q, k, v, do, csr)
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_many_work_items_all_gradients():
    """8 heads x 71 key (and query) tiles = 568 work items per backward kernel,
    several per persistent CTA on 148 SMs: every element of dQ, dK and dV
    against the dense reference, head by head."""
    wl = I.small_workload("bmany", 1, 8, 128, 9, 1000, 128, 42)
    q, k, v, do = I.draw(wl, device=DEV, backward=True)
    csr = rb.radial_mask_build(9, 1000, 128, sink=1)
    _, _, dq, dk, dv = _gpu_fwd_bwd(q, k, v, do, csr)
    x = [t[0].double().cpu().numpy() for t in (q, k, v, do)]
    ref = oracle_pool.run("bwd_head", [(x[0][h], x[1][h], x[2][h], x[3][h], 9, 1000, True) for h in range(8)])
    for h, (rq, rk, rv) in enumerate(ref):
        for name, g, r in zip(("dQ", "dK", "dV"), (dq, dk, dv), (rq, rk, rv)):
            err = np.abs(g[0, h].double().cpu().numpy() - r).max()
            assert err <= G_MAX, f"head {h}: {name} max-abs {err:.3e}"


def _large_check(name, rows_per_head, dkdv_heads, cols_per_head):
    wl = I.WORKLOADS[name]
    q, k, v, do = I.draw(wl, device=DEV, backward=True)
    csr = rb.radial_mask_build(wl.frames, wl.tokens_per_frame, wl.block, sink=1)
    o, lse, dq, dk, dv = _gpu_fwd_bwd(q, k, v, do, csr)
    # identities over all keys, per (head, feature), in fp64 on the host
    dk64 = dk.double().sum(dim=2)
    dv64 = dv.double().sum(dim=2)
    do64 = do.double().sum(dim=2)
    dk_scale = dk.double().abs().sum(dim=2)
    dv_scale = dv.double().abs().sum(dim=2)
    # bf16 storage of each term (2^-9 relative) plus the bf16 O inside rowsum(dO o O)
    assert (dk64.abs() <= 2.0 ** -7 * dk_scale + 1e-3).all(), "sum_k dK != 0"
    assert ((dv64 - do64).abs() <= 2.0 ** -7 * dv_scale + 1e-3).all(), "sum_k dV != sum_q dO"
    scale = 1.0 / np.sqrt(wl.head_dim)
    # dK / dV on sampled key columns of seeded heads: every query's LSE and
    # rowsum(dO o O) of those heads recomputed in fp64 by the reference
    rng = np.random.default_rng(3000 + wl.seed)
    for h in sorted(rng.choice(wl.heads, size=dkdv_heads, replace=False).tolist()):
        cols = A.sample_rows(wl.n, cols_per_head, wl.tokens_per_frame, wl.block, seed=4000 + h)
        hq, hk, hv, hdo = (t[0, h].double().cpu().numpy() for t in (q, k, v, do))
        lse_ref, dr_ref = A.head_row_stats(hq, hk, hv, hdo, wl.frames, wl.tokens_per_frame, True, scale)
        dk_ref, dv_ref = A.dkdv_cols(hq, hk, hv, hdo, lse_ref, dr_ref, cols, wl.frames, wl.tokens_per_frame,
                                     True, scale)
        cidx = torch.as_tensor(cols, device=DEV)
        for nm, g, r in (("dK", dk, dk_ref), ("dV", dv, dv_ref)):
            err = np.abs(g[0, h, cidx].double().cpu().numpy() - r).max()
            assert err <= G_MAX, f"{name} head {h}: {nm} max-abs {err:.3e} on {len(cols)} key columns"
        del hq, hk, hv, hdo
    # sampled dQ rows against the reference, every head
    tasks, got = [], []
    for h in range(wl.heads):
        rows = A.sample_runs(wl.n, rows_per_head, wl.tokens_per_frame, wl.block, seed=2000 + h)
        ridx = torch.as_tensor(rows, device=DEV)
        tasks.append((q[0, h, ridx].double().cpu().numpy(), k[0, h].float().cpu().numpy(),
                      v[0, h].float().cpu().numpy(), do[0, h, ridx].double().cpu().numpy(),
                      rows, wl.frames, wl.tokens_per_frame, True, scale))
        got.append(dq[0, h, ridx].float().cpu().numpy())
    ref = oracle_pool.run("dq_runs", tasks)
    err = max(np.abs(g - r).max() for g, r in zip(got, ref))
    assert err <= G_MAX, f"{name}: dQ max-abs {err:.3e}"


def test_hunyuan720p_backward_sampled():
    _large_check("hunyuan720p", int(os.environ.get("RADIAL_BWD_ROWS", "4096")), 2,
                 int(os.environ.get("RADIAL_BWD_COLS", "4096")))


@pytest.mark.slow
def test_hunyuan720p_4x_backward_sampled():
    _large_check("hunyuan720p_4x", int(os.environ.get("RADIAL_4X_BWD_ROWS", "4096")),
                 int(os.environ.get("RADIAL_4X_DKDV_HEADS", "2")), int(os.environ.get("RADIAL_4X_BWD_COLS", "4096")))
