"""Benchmark of the radial block-sparse attention hot path on B200.

Default workload: the HunyuanVideo-shaped 720p 5 s self-attention (batch 1,
24 heads, head_dim 128, 33 frames x 3600 tokens = 118,800 tokens, 128x128
tiles, attention sink on), forward call -- the shape the throughput target is
stated on.  A step is one radial_attn_fwd call over the whole batch; the
static mask is built once per shape (it depends on positions only) and its
build time is reported beside the step.  With --workload hunyuan720p_4x a
step is the 4x-length LoRA fine-tuning pass: forward plus backward.

Prints one JSON line (rank 0).  Multi-GPU (torchrun): by default the one
problem is split across the ranks by heads (rank r runs heads
[r*H/N, (r+1)*H/N) on views of the same tensors; no collective on the data
path; strong scaling); --shard replica runs one full replica per rank instead
(weak scaling).  The step time is the max over ranks.

--impl reference times the CPU reference (oracle/) on the host cores instead.
"""

from __future__ import annotations

import argparse
import json
import math
import os
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "ms and TFLOP/s (active tiles) per attention call, % of tensor peak, speedup vs dense"


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as fh:
            pk = json.load(fh)
        return float(pk["bf16_tflops"]), float(pk["bf16_tflops_sustained"]), float(pk["hbm_gbs"]), "measured"
    except Exception:
        return 1590.0, 1400.0, 6650.0, "fallback"


def _cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


# ---------------------------------------------------------------------------
# workload accounting (host-side integers only)
# ---------------------------------------------------------------------------

def tile_flops(wl, nnz, backward=False, heads=None):
    """Algorithmic flops on active tiles: 4*B^2*d per tile forward (QK^T and PV),
    10*B^2*d backward (five tile GEMMs), times batch*heads."""
    per = 4 if not backward else 10
    heads = wl.heads if heads is None else heads
    return per * wl.block * wl.block * wl.head_dim * nnz * wl.batch * heads


def allowed_pairs(frames, s, sink=True):
    """Allowed (query, key) token pairs of one head under the method's mask, by
    frame pair: the sink frame whole (s^2); a band |k - l| <= h clipped to the
    frame, s(2h+1) - h(h+1) pairs (s^2 once h >= s - 1); a sampled diagonal, s
    pairs when d is a multiple of its period c; none otherwise.  h = floor(s /
    2^r) - 1 and c = ceil(2^r / s) with r = floor(log2 max(d, 1)) (the review
    page, Sec. 4.2: Eq.4 and Fig.5)."""
    by_d = {}
    for d in range(frames):
        r = max(d, 1).bit_length() - 1
        h = (s >> r) - 1
        if h >= 0:
            hh = min(h, s - 1)
            by_d[d] = s * (2 * hh + 1) - hh * (hh + 1)
        else:
            c = -(-(1 << r) // s)
            by_d[d] = s if d % c == 0 else 0
    total = 0
    for i in range(frames):
        for j in range(frames):
            total += s * s if (sink and j == 0) else by_d[abs(i - j)]
    return total


def elem_flops(wl, pairs, heads=None):
    """Algorithmic forward flops on allowed element pairs only: 4*d per pair."""
    heads = wl.heads if heads is None else heads
    return 4 * wl.head_dim * pairs * wl.batch * heads


def whole_job_tflops(flops_per_rank, world, ms_max):
    """Whole-job throughput: every rank runs one replica of the workload
    (independent problems), so the job does world * flops_per_rank in the
    slowest rank's time."""
    return world * flops_per_rank / (ms_max * 1e-3) / 1e12


def job_tflops(flops_total, ms_max):
    """Whole-job throughput of one problem split across ranks: the problem's
    flops in the slowest rank's time."""
    return flops_total / (ms_max * 1e-3) / 1e12


def max_over_ranks(ms, world, device=None):
    """Step time as the max over ranks (all-reduce MAX; identity at world 1)."""
    if world <= 1:
        return float(ms)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(ms)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def config_of(wl, nnz):
    return {"workload": wl.name, "batch": wl.batch, "heads": wl.heads, "head_dim": wl.head_dim,
            "frames": wl.frames, "tokens_per_frame": wl.tokens_per_frame, "n_tokens": wl.n,
            "block": wl.block, "sink": True, "active_tiles": int(nnz),
            "l2": "inputs larger than L2 (no flush): Q,K,V %.2f GB per step" % (3 * wl.batch * wl.heads * wl.n * wl.head_dim * 2 / 1e9)}


# ---------------------------------------------------------------------------
# clocks sampled during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, phys_index):
        self.idx = phys_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "200",
                 "-i", str(self.idx)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def wait_first_sample(self, timeout_s=10.0):
        """Block until the sampler has printed a line (nvidia-smi's start-up
        must not overlap the timed region)."""
        t0 = time.time()
        while self.proc is not None and not self.lines and time.time() - t0 < timeout_s:
            time.sleep(0.05)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, mx, reasons, power = [], None, set(), []
        for ln in self.lines:
            p = [x.strip() for x in ln.split(",")]
            if len(p) < 9:
                continue
            try:
                sm.append(float(p[1]))
                mx = float(p[2])
                power.append(float(p[3]))
            except ValueError:
                continue
            for name, val in zip(("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"), p[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        sm.sort()
        med = sm[len(sm) // 2] if sm else None
        return {"sm_mhz": med, "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm),
                "power_w_max": max(power) if power else None}


# ---------------------------------------------------------------------------
# CPU reference timing (oracle) -- bounded sample
# ---------------------------------------------------------------------------

def oracle_rows_timing(wl, q_rows, k_head, v_head, rows, budget_s):
    """Time the CPU reference on query rows of one head; returns (seconds, rows done)."""
    from oracle import attention as A
    import numpy as np
    n = wl.n
    q = np.zeros((n, wl.head_dim))
    done, t0 = 0, time.perf_counter()
    chunk = 256
    while done < len(rows):
        r = rows[done:done + chunk]
        q[r] = q_rows[done:done + chunk]
        A.forward_rows(q, k_head, v_head, r, wl.frames, wl.tokens_per_frame, True, chunk=chunk)
        done += len(r)
        if time.perf_counter() - t0 > budget_s:
            break
    return time.perf_counter() - t0, done


def cpu_baseline(wl, nnz, q, k, v, budget_s=15.0, backward=False):
    import numpy as np
    from oracle import attention as A
    rows = A.sample_rows(wl.n, 8192, wl.tokens_per_frame, wl.block, seed=77)
    np.random.default_rng(5).shuffle(rows)
    kh = k[0, 0].float().cpu().numpy().astype(np.float64)
    vh = v[0, 0].float().cpu().numpy().astype(np.float64)
    qr = q[0, 0].float().cpu().numpy()[rows].astype(np.float64)
    secs, done = oracle_rows_timing(wl, qr, kh, vh, rows, budget_s)
    total_rows = wl.batch * wl.heads * wl.n
    full_s = secs / done * total_rows
    if backward:
        full_s *= 3.5  # forward (two products per pair) plus backward (five)
    flops = tile_flops(wl, nnz) + (tile_flops(wl, nnz, True) if backward else 0)
    return {"value": flops / full_s / 1e12, "unit": "TFLOP/s", "cores": _cores(), "kind": "oracle",
            "sample": f"{done} query rows of head 0 (fp64 NumPy forward, {secs:.1f} s), extrapolated to "
                      f"{total_rows} rows" + (" x3.5 for forward+backward" if backward else ""),
            "extrapolated_ms_per_step": full_s * 1e3}


# ---------------------------------------------------------------------------
# the GPU arm
# ---------------------------------------------------------------------------

def run_ours(args, rank, world, local_rank):
    import numpy as np
    import torch
    import torch.distributed as dist

    import block_sparse_attention_csr_b200 as rb
    from block_sparse_attention_csr_b200 import inputs as I

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    wl = I.WORKLOADS[args.workload]
    step_kind = args.step or ("fwdbwd" if wl.backward else "fwd")
    backward = step_kind != "fwd"
    peak, peak_sus, hbm, peak_src = _peaks()
    stream = torch.cuda.current_stream(dev)

    # mask: static, built once per shape
    t0 = time.perf_counter()
    csr = rb.radial_mask_build(wl.frames, wl.tokens_per_frame, wl.block, sink=1)
    mask_ms = (time.perf_counter() - t0) * 1e3
    t0 = time.perf_counter()
    csr = rb.radial_mask_build(wl.frames, wl.tokens_per_frame, wl.block, sink=1)
    mask_ms = min(mask_ms, (time.perf_counter() - t0) * 1e3)
    nnz = rb.radial_csr_info(csr)["nnz"]

    q, k, v, *rest = I.draw(wl, device=dev, backward=True)
    do = rest[0]
    heads_mode = args.shard == "heads"
    h0, h1 = (0, wl.heads)
    local = (lambda t: t)
    if heads_mode and world > 1:
        # this rank's heads of the one problem: views of the full tensors
        from block_sparse_attention_csr_b200 import sharding
        h0, h1 = sharding.head_range(wl.heads, world, rank)
        local = (lambda t: sharding.shard(t, world, rank))
    local_heads = h1 - h0
    o = local(torch.empty_like(q))
    if backward:
        dq, dk, dv = (local(torch.empty_like(t)) for t in (q, k, v))
    q, k, v, do = (local(t) for t in (q, k, v, do))
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device=dev)   # [B, local heads, N], contiguous
    if backward:
        ws = torch.empty(max(256, rb.radial_attn_bwd_workspace_size(q)), dtype=torch.uint8, device=dev)

    if step_kind == "bwd" and local_heads > 0:
        rb.radial_attn_fwd(csr, q, k, v, o=o, lse=lse, stream=stream)   # O and LSE the backward reads

    def step():
        if local_heads == 0:  # more ranks than heads: this rank has nothing to run
            return
        if step_kind != "bwd":
            rb.radial_attn_fwd(csr, q, k, v, o=o, lse=lse, stream=stream)
        if backward:
            rb.radial_attn_bwd(csr, do, q, k, v, o, lse, dq, dk, dv, ws, stream=stream)

    for _ in range(args.warmup):
        step()
    rb.radial_device_status(stream)

    phys = local_rank
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        try:
            phys = int(vis.split(",")[local_rank])
        except ValueError:
            pass
    sampler = ClockSampler(phys)

    # ---- timed region: K steps, events on the launching stream
    launches0 = rb.radial_launch_count()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    sampler.start()
    sampler.wait_first_sample()
    time.sleep(0.2)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    for a, b in evs:
        a.record(stream)
        step()
        b.record(stream)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    launches = rb.radial_launch_count() - launches0
    rb.radial_device_status(stream)
    step_ms = [a.elapsed_time(b) for a, b in evs]
    ms = float(np.mean(step_ms))
    ms_max = max_over_ranks(ms, world, dev)

    with_fwd = step_kind != "bwd"
    flops_step = (tile_flops(wl, nnz, heads=local_heads) if with_fwd else 0) + \
        (tile_flops(wl, nnz, True, local_heads) if backward else 0)
    if heads_mode:
        value = job_tflops((tile_flops(wl, nnz) if with_fwd else 0) + (tile_flops(wl, nnz, True) if backward else 0),
                           ms_max)
    else:
        value = whole_job_tflops(flops_step, world, ms_max)

    # forward kernel alone (dominant kernel of the default step) for the roofline
    fwd_ms = ms
    if backward:
        e = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(3)]
        for a, b in e:
            a.record(stream)
            rb.radial_attn_fwd(csr, q, k, v, o=o, lse=lse, stream=stream)
            b.record(stream)
        torch.cuda.synchronize(dev)
        fwd_ms = float(np.mean([a.elapsed_time(b) for a, b in e]))
    fwd_tf = tile_flops(wl, nnz, heads=local_heads) / (fwd_ms * 1e-3) / 1e12

    extra = {}
    if rank == 0 and not args.quick and world == 1:
        # dense comparator: same kernels, all-ones mask, same shape
        dcsr = rb.radial_mask_build_dense(wl.n, wl.block)
        dnnz = rb.radial_csr_info(dcsr)["nnz"]
        rb.radial_attn_fwd(dcsr, q, k, v, o=o, lse=lse, stream=stream)
        e = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(2)]
        for a, b in e:
            a.record(stream)
            rb.radial_attn_fwd(dcsr, q, k, v, o=o, lse=lse, stream=stream)
            b.record(stream)
        torch.cuda.synchronize(dev)
        dense_ms = float(np.mean([a.elapsed_time(b) for a, b in e]))
        extra["dense"] = {"fwd_ms": dense_ms, "tflops": tile_flops(wl, dnnz) / (dense_ms * 1e-3) / 1e12,
                          "speedup_radial_vs_dense_fwd": dense_ms / fwd_ms}
        del dcsr
        if not backward and not args.no_bwd:
            dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
            ws = torch.empty(rb.radial_attn_bwd_workspace_size(q), dtype=torch.uint8, device=dev)
            rb.radial_attn_bwd(csr, do, q, k, v, o, lse, dq, dk, dv, ws, stream=stream)
            e = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(2)]
            for a, b in e:
                a.record(stream)
                rb.radial_attn_bwd(csr, do, q, k, v, o, lse, dq, dk, dv, ws, stream=stream)
                b.record(stream)
            torch.cuda.synchronize(dev)
            bwd_ms = float(np.mean([a.elapsed_time(b) for a, b in e]))
            extra["bwd"] = {"ms": bwd_ms, "tflops_algorithmic": tile_flops(wl, nnz, True) / (bwd_ms * 1e-3) / 1e12,
                            "note": "10*B^2*d flops per tile (5 GEMMs); the kernels issue 7 (dQ pass recomputes S, dP)"}
            del dq, dk, dv, ws

    if rank == 0 and (args.sweep or (args.sweep is None and world == 1 and not args.quick and args.workload == "hunyuan720p")):
        extra["sweep"] = run_sweep(args, dev, stream, peak)
        extra["long_step"] = run_long_step(dev, stream, peak)

    if rank == 0 and args.lora:
        extra["lora_layer"] = run_lora_layer(wl, csr, dev, stream, args.lora_rank)

    # ---- end to end through the public API with host buffers
    e2e = None
    if rank == 0 and not args.quick and local_heads > 0:
        def pinned_like(t):
            h = torch.empty_strided(t.shape, t.stride(), dtype=t.dtype, pin_memory=True)
            h.copy_(t)
            return h

        hq, hk, hv = (pinned_like(t) for t in (q, k, v))
        hdo = do.cpu().pin_memory() if backward else None
        ho = torch.empty_strided(q.shape, q.stride(), dtype=torch.bfloat16, pin_memory=True)
        hl = torch.empty(q.shape[:3], dtype=torch.float32).pin_memory()
        if backward:
            hdq = torch.empty(q.shape, dtype=torch.bfloat16).pin_memory()
            hdk, hdv = torch.empty_like(hdq).pin_memory(), torch.empty_like(hdq).pin_memory()

        def e2e_step():
            if not backward:
                # the public host-buffer call: each group of heads is copied in
                # while the previous group's attention runs, and copied out
                # while the next one runs
                rb.radial_attn_fwd_staged(csr, hq, hk, hv, q, k, v, o_host=ho, lse_host=hl, o_dev=o, lse_dev=lse,
                                          chunks=args.e2e_chunks, stream=stream)
                return
            q.copy_(hq, non_blocking=True)
            k.copy_(hk, non_blocking=True)
            v.copy_(hv, non_blocking=True)
            if backward:
                do.copy_(hdo, non_blocking=True)
            if step_kind != "bwd":
                rb.radial_attn_fwd(csr, q, k, v, o=o, lse=lse, stream=stream)
            if backward:
                rb.radial_attn_bwd(csr, do, q, k, v, o, lse, dq, dk, dv, ws, stream=stream)
                hdq.copy_(dq, non_blocking=True)
                hdk.copy_(dk, non_blocking=True)
                hdv.copy_(dv, non_blocking=True)
            ho.copy_(o, non_blocking=True)
            hl.copy_(lse, non_blocking=True)

        e2e_step()
        torch.cuda.synchronize(dev)
        n_e2e = max(2, min(5, args.steps))
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(n_e2e):
            e2e_step()
        b.record(stream)
        torch.cuda.synchronize(dev)
        e2e_ms = a.elapsed_time(b) / n_e2e
        elt = q.numel() * 2
        h2d = 3 * elt + (elt if backward else 0)
        d2h = elt + lse.numel() * 4 + (3 * elt if backward else 0)
        e2e = {"value": (flops_step if not heads_mode else flops_step * wl.heads / local_heads) / (e2e_ms * 1e-3) / 1e12,
               "unit": "TFLOP/s", "ms_per_step": e2e_ms,
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "path": ("pinned host buffers -> radial_attn_fwd_staged (C ABI): H2D copies, attention and D2H copies "
                        "of %d head groups overlapped" % args.e2e_chunks) if not backward else
                       "pinned host -> device copies, radial_attn_fwd/bwd via the C ABI, device -> host result copies"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(wl, nnz, q, k, v, budget_s=args.cpu_budget, backward=backward)

    if rank == 0:
        pairs = allowed_pairs(wl.frames, wl.tokens_per_frame, sink=True)
        traffic = None
        tp = os.path.join(ROOT, "profiles", "fwd_traffic.json")
        if os.path.exists(tp):
            try:
                with open(tp) as fh:
                    tj = json.load(fh)
                if (tj.get("workload") == wl.name and tj.get("kernel_sha") == kernel_sha()
                        and tj.get("kernel") == fwd_kernel_name()):
                    traffic = tj.get("dram_bytes_per_launch")
            except Exception:
                traffic = None
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_max, "higher_is_better": True,
            "scaling": "strong" if heads_mode else "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded N(0,1) bf16 Q,K,V%s)" % (",dO" if backward else ""),
            "config": dict(config_of(wl, nnz), parallelism=(f"heads/{world}" if heads_mode else f"replica x{world}"),
                           heads_per_rank_max=-(-wl.heads // world) if heads_mode else wl.heads),
            "pct_of_tensor_peak": 100.0 * value / world / peak,
            "mask_build_ms": mask_ms,
            "roofline": {"bound": "tensor", "kernel": fwd_kernel_name(), "achieved": fwd_tf, "peak": peak,
                         "unit": "TFLOP/s", "frac": fwd_tf / peak, "peak_source": f"{peak_src} bf16 burst",
                         "frac_of_sustained": fwd_tf / peak_sus, "traffic": traffic,
                         "algorithmic_flops_per_launch": tile_flops(wl, nnz, heads=local_heads), "launch_ms": fwd_ms},
            "elem": {"allowed_pairs_per_head": pairs, "flops_per_launch": elem_flops(wl, pairs, heads=local_heads),
                     "achieved": elem_flops(wl, pairs, heads=local_heads) / (fwd_ms * 1e-3) / 1e12,
                     "frac": elem_flops(wl, pairs, heads=local_heads) / (fwd_ms * 1e-3) / 1e12 / peak,
                     "note": "forward flops on allowed token pairs only (4*d per pair); the tile figure above "
                             "also counts the masked lanes of PARTIAL tiles"},
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": int(launches),
            "clocks": clocks,
        }
        line.update(extra)
        print(json.dumps(line), flush=True)


def run_sweep(args, dev, stream, peak):
    """Radial forward against dense at fixed 3600 tokens/frame over the frame
    counts of the scaling sweep: active tiles vs n log2 n, ms, TFLOP/s, % of
    peak and the speedup over dense attention of the same shape (same kernels,
    all-ones mask)."""
    import numpy as np
    import torch
    import block_sparse_attention_csr_b200 as rb
    from block_sparse_attention_csr_b200 import inputs as I

    def timed(csr, q, k, v, o, lse, reps):
        for _ in range(3):  # warm-up
            rb.radial_attn_fwd(csr, q, k, v, o=o, lse=lse, stream=stream)
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
        for a, b in ev:
            a.record(stream)
            rb.radial_attn_fwd(csr, q, k, v, o=o, lse=lse, stream=stream)
            b.record(stream)
        torch.cuda.synchronize(dev)
        return float(np.median([a.elapsed_time(b) for a, b in ev]))

    out = []
    for f in (8, 16, 33, 66, 132):
        wl = I.WORKLOADS[f"sweep_f{f}"]
        q, k, v = I.draw(wl, device=dev, backward=False)
        o = torch.empty_like(q)
        lse = torch.empty(q.shape[:3], dtype=torch.float32, device=dev)
        csr = rb.radial_mask_build(wl.frames, wl.tokens_per_frame, wl.block, sink=1)
        nnz = rb.radial_csr_info(csr)["nnz"]
        ms = timed(csr, q, k, v, o, lse, 5)
        dcsr = rb.radial_mask_build_dense(wl.n, wl.block)
        dnnz = rb.radial_csr_info(dcsr)["nnz"]
        dms = timed(dcsr, q, k, v, o, lse, 2)
        tf = tile_flops(wl, nnz) / (ms * 1e-3) / 1e12
        out.append({"frames": f, "n_tokens": wl.n, "active_tiles": int(nnz), "dense_tiles": int(dnnz),
                    "tiles_per_nlog2n": nnz / (wl.n * math.log2(wl.n)), "ms": ms, "tflops": tf,
                    "pct_of_peak": 100 * tf / peak, "dense_ms": dms,
                    "dense_tflops": tile_flops(wl, dnnz) / (dms * 1e-3) / 1e12, "speedup_vs_dense": dms / ms})
        del q, k, v, o, lse, csr, dcsr
        torch.cuda.empty_cache()
    return out


def run_long_step(dev, stream, peak):
    """The 4x-length step's attention (132 frames x 3600 tokens, 24 heads, d 128:
    the shape the length-extension fine-tuning runs at): forward and backward
    times, median of three after one warm-up."""
    import numpy as np
    import torch
    import block_sparse_attention_csr_b200 as rb
    from block_sparse_attention_csr_b200 import inputs as I

    wl = I.WORKLOADS["hunyuan720p_4x"]
    q, k, v, do = I.draw(wl, device=dev, backward=True)
    o = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device=dev)
    dq, dk, dv = (torch.empty_like(q) for _ in range(3))
    ws = torch.empty(max(256, rb.radial_attn_bwd_workspace_size(q)), dtype=torch.uint8, device=dev)
    csr = rb.radial_mask_build(wl.frames, wl.tokens_per_frame, wl.block, sink=1)
    nnz = rb.radial_csr_info(csr)["nnz"]

    def timed(fn, reps=3):
        fn()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
        for a, b in ev:
            a.record(stream)
            fn()
            b.record(stream)
        torch.cuda.synchronize(dev)
        return float(np.median([a.elapsed_time(b) for a, b in ev]))

    fwd_ms = timed(lambda: rb.radial_attn_fwd(csr, q, k, v, o=o, lse=lse, stream=stream))
    bwd_ms = timed(lambda: rb.radial_attn_bwd(csr, do, q, k, v, o, lse, dq, dk, dv, ws, stream=stream))
    rb.radial_device_status(stream)
    out = {"workload": wl.name, "active_tiles": int(nnz), "fwd_ms": fwd_ms, "bwd_ms": bwd_ms,
           "step_ms": fwd_ms + bwd_ms,
           "fwd_tflops": tile_flops(wl, nnz) / (fwd_ms * 1e-3) / 1e12,
           "bwd_tflops_algorithmic": tile_flops(wl, nnz, True) / (bwd_ms * 1e-3) / 1e12,
           "fwd_pct_of_peak": 100 * tile_flops(wl, nnz) / (fwd_ms * 1e-3) / 1e12 / peak}
    del q, k, v, do, o, lse, dq, dk, dv, ws, csr
    torch.cuda.empty_cache()
    return out


def run_lora_layer(wl, csr, dev, stream, r):
    """One LoRA-adapted attention layer step (forward + backward: dx and the
    adapter gradients) at the workload's shape, hidden size heads*head_dim,
    adapter rank r: projections on the library's tensor-core GEMM, attention
    in its block-sparse kernels."""
    import numpy as np
    import torch
    from block_sparse_attention_csr_b200 import inputs as I
    from block_sparse_attention_csr_b200.lora import RadialLoRALayer

    t = I.draw_lora_layer(wl.batch, wl.heads, wl.head_dim, wl.frames, wl.tokens_per_frame, r, wl.seed + 100,
                          device=dev)
    layer = RadialLoRALayer(csr, wl.heads, {k: v for k, v in t.items() if k.startswith("W_")},
                            {k: v for k, v in t.items() if k[:2] in ("A_", "B_")}, 1.0)

    def lstep():
        y, ctx = layer.forward(t["x"])
        return layer.backward(ctx, t["dy"])

    for _ in range(2):
        lstep()
    e = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(3)]
    for a, b in e:
        a.record(stream)
        lstep()
        b.record(stream)
    torch.cuda.synchronize(dev)
    ms = float(np.mean([a.elapsed_time(b) for a, b in e]))
    C, n = wl.heads * wl.head_dim, wl.batch * wl.n
    # per projection: forward 2nC^2 + 4nCr, backward (dx, dA, dB) 2nC^2 + 8nCr
    proj_flops = 4 * (4 * n * C * C + 12 * n * C * r)
    del t, layer
    torch.cuda.empty_cache()
    return {"rank": r, "hidden": C, "ms_per_step": ms, "projection_gemm_tflop": proj_flops / 1e12,
            "path": "4 LoRA projections (radial_lora_fwd/bwd) + radial_attn_fwd/bwd, all in this library, forward + backward"}


def fwd_kernel_name():
    return "radial_fwd_pair_kernel<128>"


def kernel_sha():
    import hashlib
    h = hashlib.sha1()
    for f in ("attn_fwd.cuh", "attn_fwd_pair.cuh", "sm100_primitives.cuh", "mask_build.cuh", "radial_lib.cu"):
        with open(os.path.join(ROOT, "block_sparse_attention_csr_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:12]


# ---------------------------------------------------------------------------
# the reference arm: the CPU reference as it stands, on the host cores
# ---------------------------------------------------------------------------

def run_reference(args, rank, world):
    if rank != 0:
        return
    import numpy as np
    import torch
    from block_sparse_attention_csr_b200 import inputs as I
    from oracle import attention as A
    from oracle import mask as M

    wl = I.WORKLOADS[args.workload]
    heads_mode = args.shard == "heads"
    st = M.tile_states_intervals(wl.frames, wl.tokens_per_frame, wl.block, True)
    nnz = int((st != 0).sum())
    # one head's K, V drawn on the CPU with the same recipe's generator
    g = torch.Generator(device="cpu").manual_seed(wl.seed)
    shape = (wl.n, wl.head_dim)
    q = torch.randn(shape, generator=g).mul_(wl.value_scale).to(torch.bfloat16).double().numpy()
    k = torch.randn(shape, generator=g).mul_(wl.value_scale).to(torch.bfloat16).double().numpy()
    v = torch.randn(shape, generator=g).mul_(wl.value_scale).to(torch.bfloat16).double().numpy()
    rows_per_step = args.ref_rows
    rng = np.random.default_rng(9)
    times = []
    for s in range(args.warmup + args.steps):
        rows = np.sort(rng.choice(wl.n, rows_per_step, replace=False))
        t0 = time.perf_counter()
        A.forward_rows(q, k, v, rows, wl.frames, wl.tokens_per_frame, True)
        dt = time.perf_counter() - t0
        if s >= args.warmup:
            times.append(dt)
    per_row = float(np.mean(times)) / rows_per_step
    full_s = per_row * wl.batch * wl.heads * wl.n
    if wl.backward:
        full_s *= 3.5
    flops = tile_flops(wl, nnz) + (tile_flops(wl, nnz, True) if wl.backward else 0)
    value = flops / full_s / 1e12
    sample = (f"{rows_per_step} query rows of one head per step (fp64 NumPy), extrapolated to "
              f"{wl.batch * wl.heads * wl.n} rows" + (" x3.5 for forward+backward" if wl.backward else ""))
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": full_s * 1e3, "higher_is_better": True,
            "scaling": "strong" if heads_mode else "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": dict(config_of(wl, nnz), parallelism=(f"heads/{world}" if heads_mode else f"replica x{world}"),
                           heads_per_rank_max=-(-wl.heads // world) if heads_mode else wl.heads),
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": _cores(), "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="hunyuan720p")
    ap.add_argument("--quick", action="store_true", help="skip dense, e2e and extras")
    ap.add_argument("--no-bwd", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--ref-rows", type=int, default=512)
    ap.add_argument("--sweep", action="store_true", default=None,
                    help="add the frame-count scaling sweep (radial vs dense); on by default on one GPU")
    ap.add_argument("--no-sweep", dest="sweep", action="store_false")
    ap.add_argument("--lora", action="store_true", help="add one LoRA-adapted attention layer step (fwd+bwd)")
    ap.add_argument("--lora-rank", type=int, default=64)
    ap.add_argument("--step", default=None, choices=["fwd", "bwd", "fwdbwd"],
                    help="what one step runs (default: the workload's own: forward, or forward+backward)")
    ap.add_argument("--e2e-chunks", type=int, default=6, help="head groups of the staged host-buffer forward")
    ap.add_argument("--shard", default="heads", choices=["heads", "replica"],
                    help="multi-GPU: split the problem's heads across ranks (default) or run one replica per rank")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        args.warmup = 3

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local_rank))
    try:
        run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
