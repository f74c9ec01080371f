"""Multi-rank host logic of bench.py on CPU with gloo (world size 2): the
step time is the max over ranks, the whole-job value counts every rank's
replica, and the reference arm prints from rank 0 only."""

import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = 10.0 + 5.0 * rank
        m = bench.max_over_ranks(ms, world)
        out[rank] = (m, bench.whole_job_tflops(1e12, world, m))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_whole_job_value():
    world = 2
    port = _free_port()
    mgr = mp.Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, port, out), nprocs=world, start_method="spawn", join=True)
    assert out[0][0] == out[1][0] == 15.0
    assert abs(out[0][1] - 2 * 1e12 / 15e-3 / 1e12) < 1e-9


def test_world_one_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(7.5, 1) == 7.5
    assert abs(bench.whole_job_tflops(2e12, 1, 1000.0) - 2.0) < 1e-12


def test_reference_arm_prints_on_rank0_only():
    env = dict(os.environ, WORLD_SIZE="2", RANK="1", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "0", "--ref-rows", "8", "--workload", "tiny"],
                       env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == ""
    env["RANK"] = "0"
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "0", "--ref-rows", "8", "--workload", "tiny"],
                       env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0
    import json
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["e2e"]["h2d_bytes_per_step"] == 0
    assert line["cpu_baseline"]["kind"] == "oracle"


# ---------------------------------------------------------------------------
# head sharding of one problem (block_sparse_attention_csr_b200.sharding)
# ---------------------------------------------------------------------------

def test_head_ranges_cover_every_head_once():
    sys.path.insert(0, ROOT)
    from block_sparse_attention_csr_b200 import sharding as S
    for heads in (1, 5, 24, 40):
        for world in (1, 2, 3, 4, 8, 9):
            owned = []
            sizes = []
            for r in range(world):
                h0, h1 = S.head_range(heads, world, r)
                owned += list(range(h0, h1))
                sizes.append(h1 - h0)
            assert owned == list(range(heads)), (heads, world)
            assert max(sizes) - min(sizes) <= 1


def _shard_worker(rank, world, port, out):
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    from block_sparse_attention_csr_b200 import sharding as S
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        g = torch.Generator().manual_seed(11)
        full = torch.randn(2, 5, 7, 4, generator=g)          # [B, H, N, D], H = 5 splits 2 / 3
        local = S.shard(full, world, rank)
        assert local.data_ptr() == full[:, S.head_range(5, world, rank)[0]].data_ptr()   # a view
        assert local.stride() == full.stride()
        res = local * 3.0 + rank * 0.0                         # any per-head computation
        back = S.gather_heads(res, 5, world)
        out[rank] = (bool(torch.equal(back, full * 3.0)), tuple(local.shape))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_head_sharded_problem_reassembles_on_every_rank():
    world = 2
    port = _free_port()
    mgr = mp.Manager()
    out = mgr.dict()
    mp.start_processes(_shard_worker, args=(world, port, out), nprocs=world, start_method="spawn", join=True)
    assert out[0][0] and out[1][0]
    assert out[0][1][1] + out[1][1][1] == 5
