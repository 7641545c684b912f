"""Build the in-tree shared library ``libfp8bq.so`` for sm_100a with nvcc.

    python -m blockwise_fp8_weight_b200.build [--verbose-ptxas] [--checked]

``--checked`` builds ``libfp8bq_checked.so`` instead: the same library with
every plain global access of its kernels bounds-checked (FP8BQ_CHECKED=1).

The library links the CUDA runtime statically, so it does not depend on
which libcudart the host process (e.g. PyTorch) loaded.
"""
from __future__ import annotations

import argparse
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
SOURCES = [os.path.join(CSRC, f) for f in ("fp8bq_api.cu", "fp8bq_kernels.cu", "fp8bq_tma.cu",
                                                   "fp8bq_dequant.cu", "fp8bq_scale.cu")]
HEADERS = [os.path.join(CSRC, f) for f in ("fp8bq_internal.h", "fp8bq_device.cuh",
                                                   "fp8bq_tile.cuh")] + [
    os.path.join(ROOT, "include", "fp8bq.h")]
LIB = os.path.join(PKG, "libfp8bq.so")
LIB_CHECKED = os.path.join(PKG, "libfp8bq_checked.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-shared", "-Xcompiler", "-fPIC,-fvisibility=hidden",
         "-cudart", "static", "--expt-relaxed-constexpr",
         # IEEE division/sqrt and no flush-to-zero (nvcc's defaults, stated explicitly)
         "-prec-div=true", "-prec-sqrt=true", "-ftz=false", "-fmad=true"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def up_to_date(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(f) <= t for f in SOURCES + HEADERS)


def build(force: bool = False, verbose_ptxas: bool = False, out: str | None = None,
          defines: tuple[str, ...] = (), checked: bool = False) -> str:
    """Compile the library (to ``out``, default the in-tree path); ``defines``
    are extra -D tuning constants; ``checked`` builds the bounds-checked
    library (default path ``libfp8bq_checked.so``)."""
    lib = out or (LIB_CHECKED if checked else LIB)
    if checked:
        defines = (*defines, "FP8BQ_CHECKED=1")
    if out is None and not force and not verbose_ptxas and \
            (checked or not defines) and up_to_date(lib):
        return lib
    tmp = lib + f".tmp{os.getpid()}"
    cmd = [nvcc(), *ARCH, *FLAGS, *(f"-D{d}" for d in defines), "-I", os.path.join(ROOT, "include"),
           "-o", tmp, *SOURCES]
    if verbose_ptxas:
        cmd.insert(1, "-Xptxas=-v")
    subprocess.run(cmd, check=True)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose-ptxas", action="store_true")
    ap.add_argument("--checked", action="store_true")
    a = ap.parse_args()
    print(build(force=a.force, verbose_ptxas=a.verbose_ptxas, checked=a.checked))
    sys.exit(0)
