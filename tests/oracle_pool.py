"""Full-size oracle references for the GPU parity tests, computed in a
process pool.

Every output of a full-size GPU run is compared with the FP64 oracle, not a
sample of rows.  The oracle forms dense W one block of rows at a time, which
is slow for the 8B / 27B-shaped passes, so the references are computed by
worker processes while the GPU runs.  Each worker regenerates its matrix from
the seeded spec (``wal_synth``) and evaluates the oracle over all rows; no
worker ever sees a GPU result, and none touches CUDA: the pool is started
with the ``spawn`` method and imports only numpy, ``oracle`` and
``wal_synth``.
"""
from __future__ import annotations

import multiprocessing as mp
import os

import numpy as np

ROW_CHUNK = 2048  # rows of dense W formed at a time (2048 x 17408 x 8 B = 285 MB at most)

_POOL = None


def pool():
    """The shared spawn-started pool (one worker per host core, BLAS single-threaded)."""
    global _POOL
    if _POOL is None:
        saved = {k: os.environ.get(k) for k in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS")}
        for k in saved:
            os.environ[k] = "1"
        try:
            _POOL = mp.get_context("spawn").Pool(processes=max(1, min(os.cpu_count() or 1, 32)))
        finally:
            for k, v in saved.items():
                if v is None:
                    os.environ.pop(k, None)
                else:
                    os.environ[k] = v
    return _POOL


def _rows_in_chunks(n, fn, M):
    out = np.empty((M, n), dtype=np.float64)
    for r0 in range(0, n, ROW_CHUNK):
        rows = np.arange(r0, min(n, r0 + ROW_CHUNK))
        out[:, rows] = fn(rows)
    return out


def _v1_job(args):
    workload, spec, X = args
    import oracle
    from wal_synth import gen_matrix
    c = gen_matrix(workload, spec)
    Y = _rows_in_chunks(spec.N, lambda rows: oracle.matmul_rows(c, X, rows), X.shape[0])
    return Y, c.alpha


def _pq2_job(args):
    N, K, config_id, index, X = args
    import oracle.pq2_oracle as pq
    from wal_synth import gen_pq2
    T, d = gen_pq2(N, K, config_id, index)
    m = pq.Pq2(N, K, T, d)
    return _rows_in_chunks(N, lambda rows: pq.matmul_rows(m, X, rows), X.shape[0]), d


def _int4_job(args):
    N, K, config_id, index, X, r0, r1 = args
    import oracle.head_oracle as ho
    from wal_synth import gen_int4
    q, d = gen_int4(N, K, config_id, index)
    return ho.int4_matmul_rows(q, d, X, np.arange(r0, r1))


def v1_refs_async(workload, specs, xs):
    """Start the oracle for matrices `specs` of `workload` with activations
    xs[i] (bf16 bits [M, K]); .get() gives [(Y float64 [M, N], alpha bits)]."""
    return pool().map_async(_v1_job, [(workload, s, np.asarray(x).reshape(-1, s.K)) for s, x in zip(specs, xs)],
                            chunksize=1)


def pq2_refs_async(jobs):
    """jobs: (N, K, config_id, index, X bits [M, K]); .get() gives [(Y, d bits)]."""
    return pool().map_async(_pq2_job, jobs, chunksize=1)


def int4_ref(N, K, config_id, index, X, chunk=8192):
    """Y = X W^T of an INT4 matrix from gen_int4, all N rows, split over the pool."""
    X = np.asarray(X).reshape(-1, K)
    parts = pool().map(_int4_job, [(N, K, config_id, index, X, r0, min(N, r0 + chunk)) for r0 in range(0, N, chunk)])
    return np.concatenate(parts, axis=1)
