"""Runs oracle functions on a process pool for the full-size parity tests.

The pool uses the ``spawn`` start method, so it is safe to create after the
CUDA context exists; each worker limits its BLAS to one thread, so the pool's
processes share the host cores instead of oversubscribing them.  No method
arithmetic here: the workers only call ``oracle``.
"""

from __future__ import annotations

import multiprocessing as mp
import os


def _energy_job(args):
    from threadpoolctl import threadpool_limits

    import oracle
    q, k, N, block, scale = args
    with threadpool_limits(1):
        return oracle.block_energy(q, k, N, block, block, scale)


def block_energies(jobs):
    """oracle.block_energy of every (q [1, Np, d], k, N, block, scale) job, in job order."""
    procs = max(1, min(len(jobs), len(os.sched_getaffinity(0))))
    with mp.get_context("spawn").Pool(procs) as pool:
        return pool.map(_energy_job, jobs, chunksize=1)
