"""Runs the oracle's W4A16 GEMM on every host core.

TEST INFRASTRUCTURE ONLY, like the rest of ``oracle/``: only the CPU-baseline and reference
legs of ``bench.py`` use it. It changes nothing in the oracle's arithmetic: each worker calls
:func:`oracle.awq_oracle.gemm_w4a16` unchanged on a slice of the weight's output rows
(output rows are independent, so the slices together give exactly the full result).

Workers are spawned processes (never forked: the parent may hold a CUDA context), each
limited to one BLAS thread, one per core. The packed weights live in shared memory, so a
task is only (job, first row, last row).
"""
from __future__ import annotations

import multiprocessing as mp
import os
import platform
import sys
import time
import types
from concurrent.futures import ProcessPoolExecutor
from multiprocessing import shared_memory

import numpy as np

_W = {}   # worker side: job index -> (X1, qweight, scales, zeros, K, bits, group)


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return platform.processor() or "unknown"


def _attach(spec):
    name, shape, dtype = spec
    shm = shared_memory.SharedMemory(name=name)
    return shm, np.ndarray(shape, dtype=np.dtype(dtype), buffer=shm.buf)


def _init(job_specs):
    try:
        from threadpoolctl import threadpool_limits
        threadpool_limits(limits=1)
    except ImportError:  # pragma: no cover
        pass
    keep = []
    for j, (specs, K, bits, group) in enumerate(job_specs):
        arrs = []
        for spec in specs:
            shm, a = _attach(spec)
            keep.append(shm)
            arrs.append(a)
        _W[j] = (*arrs, K, bits, group)
    _W["shm"] = keep


def _task(j, r0, r1):
    from oracle.awq_oracle import gemm_w4a16
    X1, qw, sc, z, K, bits, group = _W[j]
    gemm_w4a16(X1, qw[r0:r1], sc[:, r0:r1], z[:, r0:r1], r1 - r0, K, bits, group)
    return r1 - r0


def _noop(_=None):
    return os.getpid()


class OracleGemmPool:
    """The oracle's gemm_w4a16 over the rows of several packed weights, on every core.

    ``jobs``: list of (X [M, K] fp16, qweight, scales [G, N], zeros [G, N], K, bits, group).
    """

    def __init__(self, jobs, cores: int | None = None):
        self.cores = int(cores or os.cpu_count() or 1)
        self._shm = []
        self._pool = None
        specs = []
        self.rows = []
        for X, qw, sc, z, K, bits, group in jobs:
            arrs = []
            for a in (np.ascontiguousarray(X), np.ascontiguousarray(qw),
                      np.ascontiguousarray(sc), np.ascontiguousarray(z)):
                shm = shared_memory.SharedMemory(create=True, size=max(a.nbytes, 1))
                np.ndarray(a.shape, a.dtype, buffer=shm.buf)[...] = a
                self._shm.append(shm)
                arrs.append((shm.name, a.shape, a.dtype.str))
            specs.append((arrs, K, bits, group))
            self.rows.append(qw.shape[0])
        try:
            self._start(specs)
        except BaseException:
            self.close()
            raise
        self._tasks = []
        for j, n in enumerate(self.rows):
            step = max(1, -(-n // self.cores))
            self._tasks += [(j, r0, min(n, r0 + step)) for r0 in range(0, n, step)]

    def _start(self, specs):
        self._pool = ProcessPoolExecutor(self.cores, mp_context=mp.get_context("spawn"),
                                         initializer=_init, initargs=(specs,))
        # Start every worker (imports, shared-memory attach) before anything is timed. A
        # spawned process normally re-runs the parent's main script first; the parent's
        # __main__ is hidden while the workers start, so they import numpy and the oracle only.
        main = sys.modules["__main__"]
        sys.modules["__main__"] = types.ModuleType("__main__")
        try:
            list(self._pool.map(_noop, range(4 * self.cores)))
        finally:
            sys.modules["__main__"] = main

    def run_once(self) -> float:
        """One pass over every row of every job; returns its wall-clock seconds."""
        t0 = time.perf_counter()
        futs = [self._pool.submit(_task, *t) for t in self._tasks]
        done = sum(f.result() for f in futs)
        assert done == sum(self.rows)
        return time.perf_counter() - t0

    def close(self):
        if getattr(self, "_pool", None) is not None:
            self._pool.shutdown()
            self._pool = None
        for shm in self._shm:
            shm.close()
            shm.unlink()
        self._shm = []
