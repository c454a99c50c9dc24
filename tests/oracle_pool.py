"""The fp64 oracle over whole workloads, every (document, head) problem in a
process pool (test infrastructure, like the oracle it calls).

``ref_attention`` computes each (document, head) independently from the
definition, so running the problems in separate processes and writing each
result into its slice gives exactly what one call over the whole pack gives.
The pool is started with the ``spawn`` method (never forked from a process
that already holds a CUDA context) and its workers run single-threaded BLAS,
so the host's cores are shared between problems rather than inside one.
"""
from __future__ import annotations

import multiprocessing as mp
import os

import numpy as np

from oracle.attention import ref_attention


def _one(args):
    q, k, v, causal, scale, row_chunk = args
    L = q.shape[0]
    out, lse = ref_attention(q, k, v, [0, L], causal, scale, row_chunk=row_chunk)
    return out[:, 0, :], lse[0]


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def full_reference(q, k, v, lengths, causal: bool, scale: float, heads=None,
                   workers: int | None = None, row_chunk: int = 1024):
    """fp64 oracle output and lse of every row of the selected heads.

    q, k, v: fp64 numpy [T, H, d] (already dequantised for the MXFP8 path);
    lengths: document lengths in pack order; heads: the heads to compute
    (default all).  Returns (out [T, len(heads), d], lse [len(heads), T])."""
    T, H, d = q.shape
    heads = list(range(H)) if heads is None else list(heads)
    starts = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    tasks, where = [], []
    for i in range(len(lengths)):
        a, b = int(starts[i]), int(starts[i + 1])
        if b == a:
            continue
        for hi, h in enumerate(heads):
            tasks.append((np.ascontiguousarray(q[a:b, h:h + 1]),
                          np.ascontiguousarray(k[a:b, h:h + 1]),
                          np.ascontiguousarray(v[a:b, h:h + 1]), causal, scale, row_chunk))
            where.append((a, b, hi))
    out = np.zeros((T, len(heads), v.shape[2]), dtype=np.float64)
    lse = np.full((len(heads), T), -np.inf, dtype=np.float64)
    n = min(workers or host_cores(), 32, max(1, len(tasks)))
    # largest problems first, so the pool does not end on a long straggler
    order = sorted(range(len(tasks)), key=lambda t: -(where[t][1] - where[t][0]))
    saved = {key: os.environ.get(key) for key in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS",
                                                  "MKL_NUM_THREADS")}
    for key in saved:
        os.environ[key] = "1"
    try:
        ctx = mp.get_context("spawn")
        with ctx.Pool(n) as pool:
            results = pool.map(_one, [tasks[t] for t in order], chunksize=1)
    finally:
        for key, val in saved.items():
            if val is None:
                os.environ.pop(key, None)
            else:
                os.environ[key] = val
    for t, (o, l_) in zip(order, results):
        a, b, hi = where[t]
        out[a:b, hi] = o
        lse[hi, a:b] = l_
    return out, lse
