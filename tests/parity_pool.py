"""Whole-tensor parity for the large workloads: the oracle runs over row chunks in a pool of
host processes, and each chunk is compared where it is computed.  The oracle's arithmetic is
unchanged; only the loop over rows is spread over the host's cores.

The pool is started with the ``spawn`` method: the test process has already initialised
CUDA, and a process forked after that can hang.  The children import numpy and the oracle
only (no torch, no CUDA), with one BLAS thread each."""

from __future__ import annotations

import multiprocessing as mp
import os
from contextlib import contextmanager

import numpy as np

CHUNK_ROWS = 256


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


@contextmanager
def oracle_pool(workers: int | None = None):
    n = max(1, min(host_cores(), 64) if workers is None else workers)
    saved = {k: os.environ.get(k) for k in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS")}
    for k in saved:
        os.environ[k] = "1"
    try:
        pool = mp.get_context("spawn").Pool(n)
    finally:
        for k, v in saved.items():
            if v is None:
                os.environ.pop(k, None)
            else:
                os.environ[k] = v
    try:
        yield pool
    finally:
        pool.close()
        pool.join()


def _amax_chunk(args):
    import oracle as o
    x, block = args
    return float(o.rotated_amax(x, block))


def _compare_chunk(args):
    import oracle as o
    from oracle.parity import compare
    x, outs, fmt, group, block, rule, ts, labels = args
    res = o.rotate_quantize(x, fmt, group, block, rule, tensor_scale=ts)
    return [compare(res, c, s, label=l) for (c, s), l in zip(outs, labels)]


def _chunks(M: int):
    return [(r, min(M, r + CHUNK_ROWS)) for r in range(0, M, CHUNK_ROWS)]


def rotated_amax(pool, x: np.ndarray, block: int) -> np.float32:
    """max |fl(y)| over the whole tensor (the oracle's rotated_amax, chunk by chunk)."""
    parts = pool.map(_amax_chunk, [(x[a:b], block) for a, b in _chunks(x.shape[0])])
    return np.float32(max(parts) if parts else 0.0)


def compare_all_rows(pool, x: np.ndarray, outs: list, labels: list, fmt: int, group: int, block: int, rule: int,
                     tensor_scale=None) -> list:
    """One merged ParityReport per entry of ``outs`` ((codes, scales) of the whole tensor),
    against the oracle on every row."""
    args = [(x[a:b], [(c[a:b], s[a:b]) for c, s in outs], fmt, group, block, rule, tensor_scale, labels)
            for a, b in _chunks(x.shape[0])]
    merged = None
    for reps in pool.imap(_compare_chunk, args, chunksize=1):
        merged = reps if merged is None else [m.merge(r) for m, r in zip(merged, reps)]
    return merged
