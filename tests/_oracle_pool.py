"""The oracle's importance-weighted fit over row chunks in worker processes (test infrastructure).

The workers are started with the spawn method, so the pool is safe to create in a process that has
already initialised CUDA.  Each worker runs the oracle unchanged on whole rows; rows are independent in
the fit, so concatenating the chunks gives exactly the single-process result.
"""
from __future__ import annotations

import concurrent.futures
import multiprocessing as mp
import os

import numpy as np

from oracle import qlinear_oracle as O


def _fit_chunk(args):
    w, imp = args
    return O.pack_imatrix(w, imp)


def pack_imatrix_parallel(w: np.ndarray, imp: np.ndarray, chunk: int = 128, workers: int | None = None):
    """O.pack_imatrix(w, imp) computed over chunks of `chunk` rows in spawned worker processes."""
    n = w.shape[0]
    workers = workers or max(1, min(16, os.cpu_count() or 1))
    jobs = [(w[i:i + chunk], imp) for i in range(0, n, chunk)]
    with concurrent.futures.ProcessPoolExecutor(max_workers=workers, mp_context=mp.get_context("spawn")) as ex:
        parts = list(ex.map(_fit_chunk, jobs))
    return (np.concatenate([p[0] for p in parts]), np.concatenate([p[1] for p in parts]),
            np.concatenate([p[2] for p in parts]))
