"""Run the oracle's decode over many sequences in a process pool.

TEST AND CPU-TIMING INFRASTRUCTURE ONLY (see the package docstring).  Used by
the CPU-baseline and reference legs of bench.py to time the oracle on the
host's cores.  Each task is one sequence with its own compact pools, so a
worker needs only numpy and this package.  The pool uses the "spawn" start
method and pins BLAS to one thread per worker.
"""

from __future__ import annotations

import multiprocessing as mp
import os
import time

import numpy as np

from .paged import decode


def _init_worker():
    for v in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS"):
        os.environ[v] = "1"


def decode_task(task):
    """task = (q_raw [1,Hq,D], q_dtype, k_raw, v_raw, cache_dtype, table [1,W],
    lens [1], scale, Hkv, k_scale, v_scale) -> (out [1,Hq,D], seconds)."""
    t0 = time.perf_counter()
    out = decode(*task)
    return out, time.perf_counter() - t0


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def run_decode_tasks(tasks, workers: int):
    """Run tasks on `workers` spawned processes; returns (outputs, wall seconds)."""
    for v in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS"):
        os.environ.setdefault(v, "1")
    ctx = mp.get_context("spawn")
    with ctx.Pool(processes=workers, initializer=_init_worker) as pool:
        pool.map(_noop, range(workers))  # start-up outside the timed region
        t0 = time.perf_counter()
        res = pool.map(decode_task, tasks, chunksize=1)
        wall = time.perf_counter() - t0
    return [r[0] for r in res], wall


def _noop(_):
    return np.zeros(1)


class OraclePool:
    """A spawned pool of ``workers`` processes (BLAS pinned to one thread
    each) kept open for several timed runs of the oracle's decode.

        with OraclePool(16) as pool:
            outs, wall = pool.run(tasks)
    """

    def __init__(self, workers: int):
        self.workers = int(workers)
        self._pool = None

    def __enter__(self):
        for v in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS"):
            os.environ.setdefault(v, "1")
        ctx = mp.get_context("spawn")
        self._pool = ctx.Pool(processes=self.workers, initializer=_init_worker)
        self._pool.map(_noop, range(self.workers))  # start-up outside any timed region
        return self

    def __exit__(self, *exc):
        self._pool.close()
        self._pool.join()
        self._pool = None
        return False

    def run(self, tasks):
        """Decode the tasks on the pool; returns (outputs, wall seconds)."""
        t0 = time.perf_counter()
        res = self._pool.map(decode_task, tasks, chunksize=1)
        return [r[0] for r in res], time.perf_counter() - t0


def cpu_model() -> str:
    """The host CPU's model name (from /proc/cpuinfo), or "unknown"."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.lower().startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:  # pragma: no cover
        pass
    return "unknown"
