"""The f64 oracle spread over the host's cores.

TEST INFRASTRUCTURE ONLY, like the oracle itself: only the tests,
``__graft_entry__.smoke()`` and the CPU-baseline / reference arm of
``bench.py`` use it.  It holds none of the method's arithmetic: it stages
input arrays in files, hands row ranges to worker processes, and each worker
calls an ``oracle.kld_oracle`` function on its rows after the same exact
conversion to float64 the tests use (bf16 bits -> f32 -> f64, f32 -> f64).

Workers are spawned (never forked), so a pool can be started after the
parent has touched a GPU, and one worker runs per host core with numpy
limited to one thread each.  Inputs cross the process boundary as file
names and row ranges only; the files live in a private temporary directory
that ``close()`` removes.
"""
from __future__ import annotations

import multiprocessing as mp
import os
import shutil
import tempfile

import numpy as np

# how each staged array is turned into the oracle's input
_KINDS = ("bf16", "f32", "f64", "int")


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def _convert(kind: str, a: np.ndarray) -> np.ndarray:
    from oracle import kld_oracle as O
    if kind == "bf16":
        return O.bf16_bits_to_f64(a)
    if kind in ("f32", "f64"):
        return O.as_f64(a)
    return np.asarray(a)


def _job(job):
    """Worker: rows [a, b) of every row-sliced staged array, converted, and
    every whole staged array, passed by keyword to the named oracle function
    with the remaining keyword arguments."""
    fn, rows, whole, kwargs, a, b = job
    from oracle import kld_oracle as O
    args = dict(kwargs)
    for name, (path, dtype, shape, kind) in rows.items():
        m = np.memmap(path, dtype=dtype, mode="r", shape=shape)
        args[name] = _convert(kind, np.array(m[a:b]))
    for name, (path, dtype, shape, kind) in whole.items():
        m = np.memmap(path, dtype=dtype, mode="r", shape=shape)
        args[name] = _convert(kind, np.array(m))
    return getattr(O, fn)(**args)


def _noop(_):
    return 0


class OraclePool:
    """A pool of spawned oracle workers, one per host core (or `cores`)."""

    def __init__(self, cores: int | None = None):
        self.cores = cores or host_cores()
        saved = os.environ.get("OMP_NUM_THREADS")
        os.environ["OMP_NUM_THREADS"] = "1"
        try:
            self.pool = mp.get_context("spawn").Pool(self.cores)
        finally:
            if saved is None:
                del os.environ["OMP_NUM_THREADS"]
            else:
                os.environ["OMP_NUM_THREADS"] = saved
        self.pool.map(_noop, range(4 * self.cores))   # every worker up before any timing
        self.dir = tempfile.mkdtemp(prefix="kld_oracle_pool_")

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()

    def stage(self, name: str, array, kind: str):
        """Write `array` (numpy, or a torch tensor: its raw bits) to a file;
        returns the handle that run() takes."""
        assert kind in _KINDS, kind
        a = _as_numpy_bits(array)
        path = os.path.join(self.dir, name)
        m = np.memmap(path, dtype=a.dtype, mode="w+", shape=a.shape if a.ndim else (1,))
        m[...] = a
        m.flush()
        del m
        return (path, a.dtype.str, a.shape if a.ndim else (1,), kind)

    def run_async(self, fn: str, rows: dict, n: int, rows_per_job: int = 4, whole: dict | None = None,
                  start: int = 0, **kwargs):
        """Start the oracle function `fn` over rows [start, start + n):
        `rows` maps its argument names to staged arrays sliced by row,
        `whole` to staged arrays passed whole, and the keyword arguments go
        as they are.  Returns an object whose get() gives the per-job results."""
        jobs = [(fn, dict(rows), dict(whole or {}), kwargs, a, min(start + n, a + rows_per_job))
                for a in range(start, start + n, rows_per_job)]
        return self.pool.map_async(_job, jobs, chunksize=1)

    def run(self, fn: str, rows: dict, n: int, rows_per_job: int = 4, whole: dict | None = None,
            start: int = 0, **kwargs) -> dict:
        """The oracle function over rows [start, start + n), results joined in row order."""
        return concat(self.run_async(fn, rows, n, rows_per_job, whole, start, **kwargs).get())

    def close(self):
        self.pool.terminate()
        self.pool.join()
        shutil.rmtree(self.dir, ignore_errors=True)


def concat(parts) -> dict:
    """Per-job result dicts joined along their first axis."""
    out = {}
    for k in parts[0]:
        vals = [p[k] for p in parts]
        out[k] = np.concatenate([np.atleast_1d(np.asarray(v)) for v in vals])
    return out


def _as_numpy_bits(array) -> np.ndarray:
    if isinstance(array, np.ndarray):
        return array
    import torch
    t = array.detach().cpu()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()
