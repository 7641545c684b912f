"""Seeded synthetic weight matrices shaped like the pages' workloads.

Input preparation only: this package draws random numbers, shapes them into
the value distributions of the workloads and rounds them to the storage type.
It holds none of the quantizer's arithmetic.  Both the CPU oracle and the CUDA
library consume the buffers it writes.

The workloads (tensor lists, value recipes and seeds) are in
``synth.workloads``; the generator itself is ``synth.c`` (SplitMix64 in
counter mode + Box-Muller, multi-threaded, order independent).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from dataclasses import dataclass, field

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "synth.c")
_LIB_PATH = os.path.join(_HERE, "libsynth.so")

DIST_NORMAL = 0
DIST_STUDENT_T3 = 1

_lock = threading.Lock()
_lib = None


class _Spec(ctypes.Structure):
    _fields_ = [
        ("seed", ctypes.c_uint64), ("tensor_id", ctypes.c_uint64),
        ("batch", ctypes.c_int64), ("M", ctypes.c_int64), ("N", ctypes.c_int64),
        ("ld", ctypes.c_int64), ("batch_stride", ctypes.c_int64),
        ("dtype", ctypes.c_int32), ("dist", ctypes.c_int32),
        ("sigma", ctypes.c_double), ("row_lognormal_sigma", ctypes.c_double),
        ("batch_lognormal_sigma", ctypes.c_double),
        ("outlier_p", ctypes.c_double), ("outlier_lo", ctypes.c_double),
        ("outlier_hi", ctypes.c_double), ("pad_value", ctypes.c_double),
        ("nthreads", ctypes.c_int32),
    ]


def build(force: bool = False) -> str:
    """Compile ``synth.c`` into ``libsynth.so`` (gcc)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    subprocess.run(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread", "-Wall",
                    "-o", tmp, _SRC, "-lm"], check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _libsynth() -> ctypes.CDLL:
    global _lib
    with _lock:
        if _lib is None:
            build()
            L = ctypes.CDLL(_LIB_PATH)
            L.synth_fill.argtypes = [ctypes.POINTER(_Spec), ctypes.c_void_p]
            L.synth_fill.restype = ctypes.c_int
            L.synth_f32_to_bf16.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p]
            L.synth_f32_to_bf16.restype = None
            _lib = L
    return _lib


@dataclass
class TensorSpec:
    """One weight tensor of a workload: [batch, M, N] with row stride ``ld``.

    ``batch > 1`` is a fused-expert tensor whose experts each get their own
    descale grid.  Values: ``dist`` (normal or Student-t with 3 degrees of
    freedom) times ``sigma``, times exp(row_lognormal_sigma * z_row) per row
    and exp(batch_lognormal_sigma * z_batch) per expert; with probability
    ``outlier_p`` an element is replaced by +-U(outlier_lo, outlier_hi).
    """
    name: str
    M: int
    N: int
    batch: int = 1
    ld: int | None = None
    dtype: str = "bf16"          # "bf16" or "f32"
    block: tuple[int, int] = (128, 128)
    seed: int = 0
    tensor_id: int = 0
    dist: int = DIST_NORMAL
    sigma: float = 0.02
    row_lognormal_sigma: float = 0.0
    batch_lognormal_sigma: float = 0.0
    outlier_p: float = 0.0
    outlier_lo: float = 0.5
    outlier_hi: float = 4.0
    pad_value: float = 3.0e4     # fills columns N..ld-1; must never reach an output
    meta: dict = field(default_factory=dict)

    @property
    def row_stride(self) -> int:
        return self.N if self.ld is None else self.ld

    @property
    def batch_stride(self) -> int:
        return self.M * self.row_stride

    @property
    def numel_storage(self) -> int:
        return self.batch * self.batch_stride

    @property
    def numel(self) -> int:
        return self.batch * self.M * self.N

    @property
    def elem_bytes(self) -> int:
        return 2 if self.dtype == "bf16" else 4

    @property
    def np_dtype(self):
        return np.uint16 if self.dtype == "bf16" else np.float32

    @property
    def grid(self) -> tuple[int, int]:
        bm, bn = self.block
        return (-(-self.M // bm), -(-self.N // bn))

    @property
    def nblocks(self) -> int:
        gm, gn = self.grid
        return self.batch * gm * gn

    @property
    def algorithmic_bytes(self) -> int:
        """Bytes the method must move: input read + e4m3 write + fp32 descales."""
        return self.numel * (self.elem_bytes + 1) + 4 * self.nblocks


def fill_into(spec: TensorSpec, ptr: int, nthreads: int | None = None) -> None:
    """Generate ``spec`` into host memory at ``ptr`` (numel_storage elements)."""
    s = _Spec(seed=spec.seed, tensor_id=spec.tensor_id, batch=spec.batch, M=spec.M,
              N=spec.N, ld=spec.row_stride, batch_stride=spec.batch_stride,
              dtype=0 if spec.dtype == "bf16" else 1, dist=spec.dist, sigma=spec.sigma,
              row_lognormal_sigma=spec.row_lognormal_sigma,
              batch_lognormal_sigma=spec.batch_lognormal_sigma,
              outlier_p=spec.outlier_p, outlier_lo=spec.outlier_lo,
              outlier_hi=spec.outlier_hi, pad_value=spec.pad_value,
              nthreads=nthreads or os.cpu_count() or 1)
    if _libsynth().synth_fill(ctypes.byref(s), ptr) != 0:
        raise ValueError(f"synth rejected spec {spec.name}")


def generate(spec: TensorSpec, nthreads: int | None = None) -> np.ndarray:
    """Generate ``spec`` as a flat numpy array (uint16 bf16 bits or float32)."""
    a = np.empty(spec.numel_storage, dtype=spec.np_dtype)
    fill_into(spec, a.ctypes.data, nthreads)
    return a


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (nearest, ties to even); returns uint16 bits."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, dtype=np.uint16)
    _libsynth().synth_f32_to_bf16(x.ctypes.data, x.size, out.ctypes.data)
    return out


def bf16_bits_to_f32(h: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to fp32 (exact)."""
    return (np.asarray(h, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)
