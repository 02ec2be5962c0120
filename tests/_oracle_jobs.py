"""Oracle evaluations for many heads at once, in spawned worker processes on
the host cores (test infrastructure: the oracle never runs on the product
path).  Spawned, not forked, because the parent process holds a CUDA context.
"""
import multiprocessing
import os


def _sparse(job):
    import numpy as np
    from oracle import calibatt_oracle as O

    q_rows, k, v, mask, block, rows = job
    # a full-length query array holding only the requested rows (the oracle
    # reads no other query row)
    q = np.zeros((k.shape[0], q_rows.shape[1]), q_rows.dtype)
    q[rows] = q_rows
    return O.block_sparse_attention(q, k, v, mask, block, rows=rows)[0]


def _anchor(job):
    from oracle import calibatt_oracle as O

    q, k, v, frames, rows_per_frame, cols, anchors, rows = job
    return O.anchor_attention(q, k, v, frames, rows_per_frame, cols, anchors, rows=rows)[0]


def _map(fn, jobs):
    cores = os.cpu_count() or 2
    workers = max(1, min(len(jobs), cores // 2))
    threads = str(max(1, cores // workers))
    saved = {k: os.environ.get(k) for k in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS")}
    for k in saved:
        os.environ[k] = threads
    try:
        with multiprocessing.get_context("spawn").Pool(workers) as pool:
            return pool.map(fn, jobs, chunksize=1)
    finally:
        for k, v in saved.items():
            if v is None:
                os.environ.pop(k, None)
            else:
                os.environ[k] = v


def sparse_rows_many(jobs):
    """[(q_rows, k, v, block_mask, block, rows)] -> [O rows], block_sparse_attention of
    each head; q_rows holds the queries of `rows` only, k and v all N keys."""
    return _map(_sparse, jobs)


def anchor_rows_many(jobs):
    """[(q, k, v, frames, rows, cols, anchors, sample_rows)] -> [O rows], anchor_attention of each head."""
    return _map(_anchor, jobs)
