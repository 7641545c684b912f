"""Builds and loads the independent e4m3fn rounding reference (e4m3_nearest.c)."""
import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "e4m3_nearest.c")
_OUT_DIR = os.path.join(_HERE, "_build")
_LIB = os.path.join(_OUT_DIR, "libe4m3_nearest.so")
_lock = threading.Lock()
_lib = None


def lib():
    global _lib
    with _lock:
        if _lib is None:
            os.makedirs(_OUT_DIR, exist_ok=True)
            if not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
                tmp = _LIB + f".tmp{os.getpid()}"
                subprocess.run(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread",
                                "-o", tmp, _SRC, "-lm"], check=True)
                os.replace(tmp, _LIB)
            L = ctypes.CDLL(_LIB)
            L.sweep.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.POINTER(ctypes.c_uint64)]
            L.sweep.restype = ctypes.c_uint64
            L.grid_values.argtypes = [ctypes.c_void_p]
            L.grid_values.restype = None
            L.nearest_codes.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p]
            L.nearest_codes.restype = None
            _lib = L
    return _lib


def grid() -> np.ndarray:
    g = np.empty(127, dtype=np.float64)
    lib().grid_values(g.ctypes.data)
    return g


def nearest_codes(v) -> np.ndarray:
    v = np.ascontiguousarray(v, dtype=np.float64)
    out = np.empty(v.shape, dtype=np.uint8)
    lib().nearest_codes(v.ctypes.data, v.size, out.ctypes.data)
    return out


def sweep(conv_fn_addr: int, nthreads: int):
    first = ctypes.c_uint64(0)
    bad = lib().sweep(conv_fn_addr, nthreads, ctypes.byref(first))
    f = first.value
    return int(bad), (f >> 16, (f >> 8) & 0xFF, f & 0xFF)
