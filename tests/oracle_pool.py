"""Run the fp64 oracle over whole heads in a pool of worker processes.

Test infrastructure (not collected by pytest: the name has no ``test_``
prefix).  The full-size parity test compares every row of every head of a
long-context workload with the oracle; one head of the 32K-key workload is a
1 TFLOP fp64 job, so the heads are spread over spawned worker processes, each
running ``oracle.attention_fp64`` unchanged on its head with a share of the
host's BLAS threads.  Workers receive the bf16 inputs and the GPU outputs of
one head (as float32, which holds bf16 exactly) and return only the error
statistics, so nothing large travels back.

The pool is created with the ``spawn`` start method: a process forked after
the parent has touched the GPU could hang.
"""

from __future__ import annotations

import multiprocessing as mp
import os

import numpy as np


def head_errors(args):
    """Worker: oracle for one (batch, head) and the errors of the GPU result.

    args = (q, k, v, o, lse, causal, scale) with q, k, v, o float32 (N, d)
    and lse float32 (N,).  Returns (max |dO|, sum dO^2, element count,
    max |dLSE|, row of the max |dO|)."""
    import oracle

    q, k, v, o, lse, causal, scale = args
    O_ref, L_ref = oracle.attention_fp64(q[None, None], k[None, None], v[None, None],
                                         causal=causal, scale=scale)
    d = np.abs(o.astype(np.float64) - O_ref[0, 0])
    e_lse = np.abs(lse.astype(np.float64) - L_ref[0, 0])
    if not (np.all(np.isfinite(d)) and np.all(np.isfinite(e_lse))):
        return float("inf"), float("inf"), d.size, float("inf"), -1
    row = int(np.unravel_index(int(np.argmax(d)), d.shape)[0])
    return float(d.max()), float(np.sum(d * d)), int(d.size), float(e_lse.max()), row


def full_errors(q, k, v, o, lse, causal: bool, scale: float, procs: int | None = None):
    """Errors of (o, lse) against the oracle over every head.

    q, k, v, o: float32 numpy arrays (BH, N, d); lse: float32 (BH, N).
    Returns a dict with max_abs, rms, max_lse, the worst head and row, and
    the worker layout used."""
    BH = q.shape[0]
    cores = os.cpu_count() or 1
    if procs is None:
        procs = max(1, min(8, cores // 2, BH))
    threads = max(1, cores // procs)
    saved = {key: os.environ.get(key) for key in ("OPENBLAS_NUM_THREADS", "OMP_NUM_THREADS",
                                                  "MKL_NUM_THREADS")}
    for key in saved:
        os.environ[key] = str(threads)
    try:
        ctx = mp.get_context("spawn")
        with ctx.Pool(procs) as pool:
            jobs = ((q[i], k[i], v[i], o[i], lse[i], causal, scale) for i in range(BH))
            res = pool.map(head_errors, jobs, chunksize=1)
    finally:
        for key, val in saved.items():
            if val is None:
                os.environ.pop(key, None)
            else:
                os.environ[key] = val
    worst = int(np.argmax([r[0] for r in res]))
    sq = sum(r[1] for r in res)
    n = sum(r[2] for r in res)
    return {
        "max_abs": max(r[0] for r in res),
        "rms": float(np.sqrt(sq / n)),
        "max_lse": max(r[3] for r in res),
        "worst_head": worst,
        "worst_row": res[worst][4],
        "procs": procs,
        "threads_per_proc": threads,
    }
