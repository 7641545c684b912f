"""CPU oracle for the blockwise FP8 (float8_e4m3fn) weight quantizer.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
benchmark's ``cpu_baseline`` / reference legs are the only callers.  The
product library never imports this package and this package never imports
the product library.

The arithmetic lives in ``fp8bq_oracle.c`` (plain single-threaded C, IEEE
binary32 round-to-nearest, no FMA contraction, no flush-to-zero); this module
builds it with gcc and marshals numpy arrays into it.  It follows the verl
documentation page "fp8_kernel.py -- FP8 量化内核", section 2 "Triton 实现"
(absmax with an eps floor, scale = absmax / 448, y = clamp(x * (1 / scale)),
fp8 store, scale store) and section 1 "统一入口" for the (fp8_data, descale)
contract.

bf16 arrays are passed as ``numpy.uint16`` holding the bf16 bit patterns.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "fp8bq_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")

#: The eps floor the library uses (the pages print the floor, not its value).
EPS = np.float32(1e-10)
#: Largest finite float8_e4m3fn value.
E4M3_MAX = 448.0

DTYPE_BF16 = 0
DTYPE_F32 = 1

_CFLAGS = ["-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
           "-fno-fast-math", "-fexcess-precision=standard", "-Wall", "-Wextra"]

_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile ``fp8bq_oracle.c`` into ``liboracle.so`` (gcc)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    subprocess.run(["gcc", *_CFLAGS, "-o", tmp, _SRC], check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def lib() -> ctypes.CDLL:
    global _lib
    with _lock:
        if _lib is None:
            build()
            L = ctypes.CDLL(_LIB_PATH)
            i64, vp, f32 = ctypes.c_int64, ctypes.c_void_p, ctypes.c_float
            L.fp8bq_oracle_e4m3.argtypes = [f32]
            L.fp8bq_oracle_e4m3.restype = ctypes.c_uint8
            L.fp8bq_oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
            L.fp8bq_oracle_e4m3_decode.restype = f32
            L.fp8bq_oracle_block.argtypes = [vp, ctypes.c_int, i64, i64, i64, ctypes.c_int,
                                             ctypes.c_int, f32, i64, i64, vp, i64, vp]
            L.fp8bq_oracle_block.restype = None
            L.fp8bq_oracle_quantize.argtypes = [vp, ctypes.c_int, i64, i64, i64, ctypes.c_int,
                                                ctypes.c_int, f32, vp, vp]
            L.fp8bq_oracle_quantize.restype = ctypes.c_int
            L.fp8bq_oracle_e4m3_array.argtypes = [vp, i64, vp]
            L.fp8bq_oracle_e4m3_array.restype = None
            L.fp8bq_oracle_e4m3_decode_array.argtypes = [vp, i64, vp]
            L.fp8bq_oracle_e4m3_decode_array.restype = None
            L.fp8bq_oracle_dequantize.argtypes = [vp, vp, i64, i64, ctypes.c_int, ctypes.c_int, vp]
            L.fp8bq_oracle_dequantize.restype = None
            L.fp8bq_oracle_dequantize_bf16.argtypes = [vp, vp, i64, i64, ctypes.c_int,
                                                       ctypes.c_int, vp]
            L.fp8bq_oracle_dequantize_bf16.restype = None
            L.fp8bq_oracle_tensor_scale.argtypes = [vp, ctypes.c_int, i64, f32]
            L.fp8bq_oracle_tensor_scale.restype = f32
            L.fp8bq_oracle_bf16.argtypes = [f32]
            L.fp8bq_oracle_bf16.restype = ctypes.c_uint16
            _lib = L
    return _lib


def _ptr(a: np.ndarray) -> int:
    return a.ctypes.data


def _dtype_code(x: np.ndarray) -> int:
    if x.dtype == np.uint16:
        return DTYPE_BF16
    if x.dtype == np.float32:
        return DTYPE_F32
    raise TypeError(f"oracle input must be uint16 (bf16 bits) or float32, got {x.dtype}")


def _check_extent(x: np.ndarray, M: int, N: int, ld: int) -> None:
    if not x.flags.c_contiguous:
        raise ValueError("oracle input must be a C-contiguous buffer")
    need = 0 if M == 0 or N == 0 else (M - 1) * ld + N
    if x.size < need:
        raise ValueError(f"input holds {x.size} elements, needs {need}")


def e4m3(v) -> np.ndarray:
    """fp32 -> float8_e4m3fn codes (RNE, saturating), element-wise."""
    v = np.ascontiguousarray(v, dtype=np.float32)
    out = np.empty(v.shape, dtype=np.uint8)
    lib().fp8bq_oracle_e4m3_array(_ptr(v), v.size, _ptr(out))
    return out


def e4m3_decode(q) -> np.ndarray:
    """float8_e4m3fn codes -> fp32 values (exact), element-wise."""
    q = np.ascontiguousarray(q, dtype=np.uint8)
    out = np.empty(q.shape, dtype=np.float32)
    lib().fp8bq_oracle_e4m3_decode_array(_ptr(q), q.size, _ptr(out))
    return out


def grid_shape(M: int, N: int, bm: int, bn: int) -> tuple[int, int]:
    return (-(-M // bm), -(-N // bn))


def quantize(x: np.ndarray, M: int, N: int, ld: int | None = None, bm: int = 128,
             bn: int = 128, eps: float = EPS) -> tuple[np.ndarray, np.ndarray]:
    """Quantize one [M, N] matrix (row stride ``ld``) block by block.

    Returns ``(y, s)``: ``y`` uint8 [M, N] e4m3fn codes, ``s`` float32
    [ceil(M/bm), ceil(N/bn)] descales.
    """
    ld = N if ld is None else ld
    _check_extent(x, M, N, ld)
    gm, gn = grid_shape(M, N, bm, bn)
    y = np.empty((M, N), dtype=np.uint8)
    s = np.empty((gm, gn), dtype=np.float32)
    rc = lib().fp8bq_oracle_quantize(_ptr(x), _dtype_code(x), M, N, ld, bm, bn,
                                     float(eps), _ptr(y), _ptr(s))
    if rc != 0:
        raise ValueError("oracle rejected the arguments")
    return y, s


def quantize_block(x: np.ndarray, M: int, N: int, ld: int | None, bm: int, bn: int,
                   bi: int, bj: int, eps: float = EPS) -> tuple[np.ndarray, float]:
    """Quantize the single block (bi, bj); returns (codes [rows, cols], descale)."""
    ld = N if ld is None else ld
    _check_extent(x, M, N, ld)
    rows = min(bm, M - bi * bm)
    cols = min(bn, N - bj * bn)
    if rows <= 0 or cols <= 0:
        raise IndexError("block outside the matrix")
    y = np.empty((rows, cols), dtype=np.uint8)
    s = np.empty(1, dtype=np.float32)
    lib().fp8bq_oracle_block(_ptr(x), _dtype_code(x), M, N, ld, bm, bn, float(eps),
                             bi, bj, _ptr(y), cols, _ptr(s))
    return y, float(s[0])


def dequantize(y: np.ndarray, s: np.ndarray, bm: int, bn: int, out_dtype: str = "f32"):
    """x_hat = dec(y) * s per block: one fp32 multiply; ``out_dtype`` "f32"
    returns float32, "bf16" returns uint16 bf16 bits (the fp32 product
    rounded to nearest even)."""
    y = np.ascontiguousarray(y, dtype=np.uint8)
    s = np.ascontiguousarray(s, dtype=np.float32)
    M, N = y.shape
    gm, gn = grid_shape(M, N, bm, bn)
    if s.size < gm * gn:
        raise ValueError("descale grid too small")
    if out_dtype == "f32":
        out = np.empty((M, N), dtype=np.float32)
        lib().fp8bq_oracle_dequantize(_ptr(y), _ptr(s), M, N, bm, bn, _ptr(out))
    elif out_dtype == "bf16":
        out = np.empty((M, N), dtype=np.uint16)
        lib().fp8bq_oracle_dequantize_bf16(_ptr(y), _ptr(s), M, N, bm, bn, _ptr(out))
    else:
        raise ValueError(out_dtype)
    return out


def tensor_scale(x: np.ndarray, eps: float = EPS) -> np.float32:
    """Per-tensor scale max(max|x|, eps) / 448 of a whole array (bf16 bits or fp32)."""
    x = np.ascontiguousarray(x)
    return np.float32(lib().fp8bq_oracle_tensor_scale(_ptr(x), _dtype_code(x), x.size, float(eps)))
