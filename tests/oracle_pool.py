"""Parallel evaluation of the CPU reference over heads (test helper).

Work is split per (batch, head) across a 'spawn' process pool so that the
fp64 reference finishes in seconds at the large shapes.  Only the CPU
reference is executed in the workers; inputs come from the seeded generators
and are passed in as float64 arrays.
"""

import multiprocessing as mp
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _init_worker(threads):
    os.environ["OPENBLAS_NUM_THREADS"] = str(threads)
    os.environ["OMP_NUM_THREADS"] = str(threads)
    if ROOT not in sys.path:
        sys.path.insert(0, ROOT)


def _fwd_rows(args):
    from oracle import attention as A
    q_rows, k, v, rows, f, s, sink, scale = args
    n = k.shape[0]
    q = np.zeros((n, k.shape[1]))
    q[rows] = q_rows
    return A.forward_rows(q, k, v, rows, f, s, sink, scale)


def _dq_rows(args):
    from oracle import attention as A
    q_rows, k, v, do_rows, rows, f, s, sink, scale = args
    n = k.shape[0]
    q = np.zeros((n, k.shape[1]))
    do = np.zeros((n, k.shape[1]))
    q[rows] = q_rows
    do[rows] = do_rows
    return A.dq_rows(q, k, v, do, rows, f, s, sink, scale)


def _fwd_runs(args):
    from oracle import attention as A
    q_rows, k, v, rows, f, s, sink, scale = args
    n = k.shape[0]
    q = np.zeros((n, k.shape[1]))
    q[rows] = q_rows
    return A.forward_runs(q, k, v, rows, f, s, sink, scale)


def _dq_runs(args):
    from oracle import attention as A
    q_rows, k, v, do_rows, rows, f, s, sink, scale = args
    n = k.shape[0]
    q = np.zeros((n, k.shape[1]))
    do = np.zeros((n, k.shape[1]))
    q[rows] = q_rows
    do[rows] = do_rows
    return A.dq_runs(q, k, v, do, rows, f, s, sink, scale)


def _bwd_head(args):
    """Forward and backward of one whole (batch, head) by the dense reference."""
    from oracle import attention as A
    from oracle import mask as M
    q, k, v, do, f, s, sink = args
    scale = 1.0 / np.sqrt(q.shape[1])
    allowed = M.token_mask(f, s, sink)
    o, lse = A.forward(q, k, v, allowed, scale)
    return A.backward(q, k, v, o, do, lse, allowed, scale)


def cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def run(fn_name, tasks, workers=None):
    fn = {"fwd_rows": _fwd_rows, "dq_rows": _dq_rows, "fwd_runs": _fwd_runs, "dq_runs": _dq_runs,
          "bwd_head": _bwd_head}[fn_name]
    if not tasks:
        return []
    c = cores()
    workers = workers or max(1, min(len(tasks), c // 2 if c > 2 else 1))
    threads = max(1, c // workers)
    if workers == 1:
        _init_worker(threads)
        return [fn(t) for t in tasks]
    # Spawned workers import NumPy (and size the BLAS thread pool) before any
    # initializer runs, so the limits go into the environment they inherit.
    saved = {k: os.environ.get(k) for k in ("PYTHONPATH", "OPENBLAS_NUM_THREADS", "OMP_NUM_THREADS")}
    env_pp = saved["PYTHONPATH"] or ""
    if ROOT not in env_pp.split(os.pathsep):
        os.environ["PYTHONPATH"] = ROOT + (os.pathsep + env_pp if env_pp else "")
    os.environ["OPENBLAS_NUM_THREADS"] = str(threads)
    os.environ["OMP_NUM_THREADS"] = str(threads)
    try:
        ctx = mp.get_context("spawn")
        with ctx.Pool(workers, initializer=_init_worker, initargs=(threads,)) as pool:
            return pool.map(fn, tasks, chunksize=1)
    finally:
        for k, v in saved.items():
            if v is None:
                os.environ.pop(k, None)
            else:
                os.environ[k] = v
