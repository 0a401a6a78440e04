"""The oracle's blocked GPTQ sweep over chunks of rows, on the host cores.

Test infrastructure (imports only NumPy and the oracle).  The listing's loop
is row-wise given U: no row reads another, so rows can be swept in chunks and
the results concatenated (the same arithmetic per row; only the rounding order
inside the BLAS block products may differ with the chunk's row count, ~1e-15
relative; pinned in test_oracle_properties).  At 28672 columns one chunk of 512 rows keeps its
block of working columns in cache, and the chunks run in a pool of worker
processes started with ``spawn`` (never forked from a process that has used
the GPU), each with one BLAS thread, U and W mapped read-only from files.
"""
from __future__ import annotations

import multiprocessing as mp
import os
import shutil
import tempfile

import numpy as np

_BLAS_VARS = ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS")


def _chunk(u_path: str, w_path: str, r0: int, r1: int, bits: int, g: int):
    from oracle.gptq import gptq_sweep_blocked_ref
    U = np.load(u_path, mmap_mode="r")
    W = np.load(w_path, mmap_mode="r")
    return gptq_sweep_blocked_ref(np.array(W[r0:r1]), U, bits, g)


def sweep_rows(Wp: np.ndarray, U: np.ndarray, bits: int, g: int, chunk: int = 512,
               workers: int | None = None):
    """(codes, scales, v) of the oracle's blocked sweep of every row of Wp."""
    from oracle.gptq import gptq_sweep_blocked_ref
    n = Wp.shape[0]
    starts = list(range(0, n, chunk))
    workers = min(len(starts), workers or len(os.sched_getaffinity(0)))
    if workers <= 1:
        parts = [gptq_sweep_blocked_ref(Wp[r:r + chunk], U, bits, g) for r in starts]
        return tuple(np.concatenate([p[i] for p in parts]) for i in range(3))
    need = U.nbytes + Wp.nbytes + (1 << 30)
    base = "/dev/shm" if os.path.isdir("/dev/shm") and \
        shutil.disk_usage("/dev/shm").free > need else None
    old = {k: os.environ.get(k) for k in _BLAS_VARS}
    with tempfile.TemporaryDirectory(dir=base) as d:
        u_path, w_path = os.path.join(d, "U.npy"), os.path.join(d, "W.npy")
        np.save(u_path, U)
        np.save(w_path, np.ascontiguousarray(Wp))
        try:
            for k in _BLAS_VARS:  # the spawned workers inherit one BLAS thread each
                os.environ[k] = "1"
            with mp.get_context("spawn").Pool(workers) as pool:
                parts = pool.starmap(_chunk, [(u_path, w_path, r, min(n, r + chunk), bits, g)
                                              for r in starts])
        finally:
            for k, v in old.items():
                if v is None:
                    os.environ.pop(k, None)
                else:
                    os.environ[k] = v
    return tuple(np.concatenate([p[i] for p in parts]) for i in range(3))
