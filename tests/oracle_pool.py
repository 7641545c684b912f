"""Full-size oracle parity: the CPU oracle over every matrix of a workload, run
in a pool of spawned worker processes, against GPU outputs copied into shared
host memory.

Test infrastructure.  The oracle stays what it is (plain, single-threaded C,
one matrix per call); the pool only runs many such calls side by side, one
matrix (or a run of experts of one stack) per task.  Inputs, GPU codes and GPU
descales live in files under /dev/shm, so a task carries offsets, not data.

The pool is started with the "spawn" method: a worker forked from a process
that has already initialised CUDA can hang.
"""
from __future__ import annotations

import multiprocessing as mp
import os
import tempfile
from dataclasses import dataclass

import numpy as np


def shm_dir() -> str:
    return "/dev/shm" if os.path.isdir("/dev/shm") else tempfile.gettempdir()


class ShmBuffer:
    """A byte buffer backed by a file in /dev/shm (visible to the workers)."""

    _count = 0

    def __init__(self, nbytes: int, tag: str):
        ShmBuffer._count += 1
        self.path = os.path.join(shm_dir(),
                                 f"fp8bq_test_{os.getpid()}_{ShmBuffer._count}_{tag}.bin")
        self.nbytes = max(int(nbytes), 1)
        self.mm = np.memmap(self.path, dtype=np.uint8, mode="w+", shape=(self.nbytes,))

    @property
    def ptr(self) -> int:
        return self.mm.ctypes.data

    def close(self) -> None:
        if self.mm is not None:
            self.mm.flush()
            del self.mm
            self.mm = None
        try:
            os.remove(self.path)
        except OSError:
            pass


@dataclass
class Task:
    """Matrices b0..b1-1 of one tensor: input, GPU codes and GPU descales are
    at the given byte offsets of their shared files (matrix b at offset +
    b * the batch stride)."""
    name: str
    b0: int
    b1: int
    M: int
    N: int
    ld: int
    bm: int
    bn: int
    dtype: str          # "bf16" or "f32"
    x_path: str
    x_off: int          # bytes
    x_bstride: int      # bytes between matrices
    y_path: str
    y_off: int
    s_path: str
    s_off: int


def _view(path: str, off: int, nbytes: int) -> np.ndarray:
    mm = np.memmap(path, dtype=np.uint8, mode="r")
    return np.array(mm[off:off + nbytes])  # a private copy: the file may be reused later


def verify(t: Task) -> tuple[str, int, int, int, str]:
    """Run the oracle on every matrix of the task and compare it with the GPU
    output bit for bit.  Returns (name, matrices, bad codes, bad descales,
    description of the first difference or "")."""
    import oracle
    es = 2 if t.dtype == "bf16" else 4
    npd = np.uint16 if t.dtype == "bf16" else np.float32
    gm, gn = -(-t.M // t.bm), -(-t.N // t.bn)
    xn = ((t.M - 1) * t.ld + t.N) * es
    bad_y = bad_s = 0
    first = ""
    for b in range(t.b0, t.b1):
        x = _view(t.x_path, t.x_off + b * t.x_bstride, xn).view(npd)
        yw, sw = oracle.quantize(x, t.M, t.N, t.ld, t.bm, t.bn)
        yg = _view(t.y_path, t.y_off + b * t.M * t.N, t.M * t.N).reshape(t.M, t.N)
        sg = _view(t.s_path, t.s_off + b * gm * gn * 4, gm * gn * 4).view(np.uint32)
        dy = np.flatnonzero(yg.reshape(-1) != yw.reshape(-1))
        ds = np.flatnonzero(sg != sw.reshape(-1).view(np.uint32))
        if (dy.size or ds.size) and not first:
            if dy.size:
                r, c = divmod(int(dy[0]), t.N)
                first = (f"matrix {b} element ({r}, {c}): got {int(yg[r, c]):#04x} "
                         f"want {int(yw[r, c]):#04x}")
            else:
                i = int(ds[0])
                first = (f"matrix {b} descale {divmod(i, gn)}: got {int(sg[i]):#010x} "
                         f"want {int(sw.reshape(-1).view(np.uint32)[i]):#010x}")
        bad_y += int(dy.size)
        bad_s += int(ds.size)
    return t.name, t.b1 - t.b0, bad_y, bad_s, first


def tasks_for(specs, x_path, x_offs, y_path, y_offs, s_path, s_offs,
              experts_per_task: int = 16) -> list[Task]:
    """One task per plain matrix; expert stacks split into runs of experts."""
    out = []
    for sp, xo, yo, so in zip(specs, x_offs, y_offs, s_offs):
        step = experts_per_task if sp.batch > 1 else 1
        for b0 in range(0, sp.batch, step):
            out.append(Task(sp.name, b0, min(sp.batch, b0 + step), sp.M, sp.N, sp.row_stride,
                            sp.block[0], sp.block[1], sp.dtype, x_path, xo,
                            sp.batch_stride * sp.elem_bytes, y_path, yo, s_path, so))
    return out


def workers() -> int:
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:
        return max(1, os.cpu_count() or 1)


class Pool:
    """A pool of spawned worker processes (the oracle library is built first,
    so the workers only load it).  A worker that dies breaks the pool and
    every pending result raises, instead of waiting for good."""

    def __init__(self, n: int | None = None):
        from concurrent.futures import ProcessPoolExecutor
        import oracle
        oracle.lib()
        self.ex = ProcessPoolExecutor(max_workers=n or workers(),
                                      mp_context=mp.get_context("spawn"))

    def map_async(self, fn, items) -> "Pending":
        return Pending([self.ex.submit(fn, it) for it in items])

    def map(self, fn, items, timeout: float = 1800.0) -> list:
        return self.map_async(fn, items).get(timeout)

    def close(self) -> None:
        self.ex.shutdown(wait=True, cancel_futures=True)


class Pending:
    def __init__(self, futures):
        self.futures = futures

    def get(self, timeout: float = 1800.0) -> list:
        import time
        end = time.monotonic() + timeout
        return [f.result(timeout=max(1.0, end - time.monotonic())) for f in self.futures]


def make_pool(n: int | None = None) -> Pool:
    return Pool(n)


def summarize(results) -> tuple[int, list[str]]:
    """(matrices checked, messages for every task with a difference)."""
    n = 0
    errs = []
    for name, mats, by, bs, first in results:
        n += mats
        if by or bs:
            errs.append(f"{name}: {by} codes and {bs} descales differ; first: {first}")
    return n, errs
