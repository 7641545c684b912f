"""Blockwise FP8 (float8_e4m3fn) weight quantizer for NVIDIA B200 (sm_100a).

A thin ctypes binding of the C ABI in ``include/fp8bq.h`` (library
``libfp8bq.so``, built in-tree by ``blockwise_fp8_weight_b200.build``).  The
functions named ``fp8bq_*`` mirror the C entry points one to one and only
marshal arguments; every step of the quantization runs in the library's CUDA
kernels.  There is no CPU or PyTorch fallback: if the library cannot be
loaded, every call raises.

On top of the raw entry points, two conveniences keep the call shapes of the
pages' Python API (verl docs "fp8_kernel.py -- FP8 量化内核", section 1 and
"vllm_fp8_utils.py", section 3):

    scaled_fp8_blockwise(data_hp, weight_block_size) -> (fp8_data, descale)
    quant_weights(named_weights, weight_block_size)  -> [(name, fp8), (name + "_scale_inv", s), ...]

They allocate the outputs with PyTorch (device memory and streams are
PyTorch's job here) and hand the pointers to the library.

With the environment variable ``FP8BQ_CHECKED=1`` set before the first call,
the process loads ``libfp8bq_checked.so`` instead: the same library with every
plain global access of its kernels bounds-checked (``fp8bq_checked_build``,
``fp8bq_debug_take_bounds``).
"""
from __future__ import annotations

import ctypes
import os
import threading
from typing import Iterable, Sequence

_PKG = os.path.dirname(os.path.abspath(__file__))
CHECKED = os.environ.get("FP8BQ_CHECKED", "0") not in ("", "0")
LIB_PATH = os.path.join(_PKG, "libfp8bq_checked.so" if CHECKED else "libfp8bq.so")

# fp8bq_dtype
FP8BQ_BF16 = 0
FP8BQ_F32 = 1
# fp8bq_status
FP8BQ_OK = 0
FP8BQ_ERR_NULL = 1
FP8BQ_ERR_SHAPE = 2
FP8BQ_ERR_BLOCK = 3
FP8BQ_ERR_DTYPE = 4
FP8BQ_ERR_OVERLAP = 5
FP8BQ_ERR_DEVICE = 6
FP8BQ_ERR_DEVICE_TIMEOUT = 7
FP8BQ_ERR_ALIGN = 8
FP8BQ_ERR_ARG = 9
FP8BQ_ERR_DEVICE_UNSAFE = 10
FP8BQ_ERR_DEVICE_BOUNDS = 11
# fp8bq_path
FP8BQ_PATH_AUTO = 0
FP8BQ_PATH_VECTOR = 1
FP8BQ_PATH_TMA = 2
FP8BQ_PATH_GENERIC = 3
FP8BQ_INJECT_DROP_FIRST_LOAD = 1
FP8BQ_INJECT_TRIM_OUTPUTS = 2

DEFAULT_BLOCK = (128, 128)


class fp8bq_desc(ctypes.Structure):
    """Mirror of ``struct fp8bq_desc`` (96 bytes)."""
    _fields_ = [
        ("x", ctypes.c_void_p),
        ("y_u8", ctypes.c_void_p),
        ("descale_f32", ctypes.c_void_p),
        ("M", ctypes.c_int64), ("N", ctypes.c_int64), ("ld", ctypes.c_int64),
        ("batch", ctypes.c_int64),
        ("x_batch_stride", ctypes.c_int64),
        ("y_batch_stride", ctypes.c_int64),
        ("s_batch_stride", ctypes.c_int64),
        ("dtype_in", ctypes.c_int32),
        ("block_m", ctypes.c_int32), ("block_n", ctypes.c_int32),
        ("reserved", ctypes.c_int32),
    ]


class fp8bq_dequant_desc(ctypes.Structure):
    """Mirror of ``struct fp8bq_dequant_desc`` (80 bytes)."""
    _fields_ = [
        ("y_u8", ctypes.c_void_p),
        ("descale_f32", ctypes.c_void_p),
        ("out", ctypes.c_void_p),
        ("batch", ctypes.c_int64), ("M", ctypes.c_int64), ("N", ctypes.c_int64),
        ("ld_out", ctypes.c_int64),
        ("out_batch_stride", ctypes.c_int64),
        ("dtype_out", ctypes.c_int32),
        ("block_m", ctypes.c_int32), ("block_n", ctypes.c_int32),
        ("reserved", ctypes.c_int32),
    ]


class fp8bq_scale_desc(ctypes.Structure):
    """Mirror of ``struct fp8bq_scale_desc`` (24 bytes)."""
    _fields_ = [("x", ctypes.c_void_p), ("numel", ctypes.c_int64),
                ("dtype_in", ctypes.c_int32), ("reserved", ctypes.c_int32)]


class Fp8bqError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = status
        msg = fp8bq_status_string(status)
        super().__init__(f"{what}: {msg}" if what else msg)


_lock = threading.Lock()
_lib = None


def lib() -> ctypes.CDLL:
    """Load ``libfp8bq.so`` (``libfp8bq_checked.so`` under FP8BQ_CHECKED=1),
    building it first with nvcc if it is missing or older than its sources.
    Raises if it cannot be built or loaded."""
    global _lib
    with _lock:
        if _lib is None:
            from . import build as _build
            if not _build.up_to_date(LIB_PATH):
                _build.build(checked=CHECKED)
            L = ctypes.CDLL(LIB_PATH)
            vp, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
            L.fp8bq_quantize.argtypes = [vp, i32, i64, i64, i64, i32, i32, vp, vp, vp]
            L.fp8bq_quantize.restype = i32
            L.fp8bq_quantize_batched.argtypes = [ctypes.POINTER(fp8bq_desc), i32, vp]
            L.fp8bq_quantize_batched.restype = i32
            L.fp8bq_dequantize.argtypes = [vp, vp, i64, i64, i64, i32, i32, vp, i32, i64, i64, vp]
            L.fp8bq_dequantize.restype = i32
            L.fp8bq_dequantize_batched.argtypes = [ctypes.POINTER(fp8bq_dequant_desc), i32, vp]
            L.fp8bq_dequantize_batched.restype = i32
            L.fp8bq_tensor_scale.argtypes = [ctypes.POINTER(fp8bq_scale_desc), i32, vp, vp]
            L.fp8bq_tensor_scale.restype = i32
            L.fp8bq_status_string.argtypes = [i32]
            L.fp8bq_status_string.restype = ctypes.c_char_p
            L.fp8bq_sync_status.argtypes = [vp]
            L.fp8bq_sync_status.restype = i32
            L.fp8bq_version.argtypes = []
            L.fp8bq_version.restype = i32
            L.fp8bq_set_path.argtypes = [i32]
            L.fp8bq_set_path.restype = i32
            L.fp8bq_get_path.argtypes = []
            L.fp8bq_get_path.restype = i32
            L.fp8bq_set_pdl.argtypes = [i32]
            L.fp8bq_set_pdl.restype = i32
            L.fp8bq_get_pdl.argtypes = []
            L.fp8bq_get_pdl.restype = i32
            L.fp8bq_path_for.argtypes = [ctypes.POINTER(fp8bq_desc)]
            L.fp8bq_path_for.restype = i32
            L.fp8bq_launch_count.argtypes = [ctypes.POINTER(fp8bq_desc), i32]
            L.fp8bq_launch_count.restype = i32
            L.fp8bq_debug_set_wait_limit_ns.argtypes = [ctypes.c_uint64]
            L.fp8bq_debug_set_wait_limit_ns.restype = i32
            L.fp8bq_debug_set_inject.argtypes = [ctypes.c_uint32]
            L.fp8bq_debug_set_inject.restype = i32
            L.fp8bq_checked_build.argtypes = []
            L.fp8bq_checked_build.restype = i32
            L.fp8bq_debug_take_bounds.argtypes = [ctypes.POINTER(ctypes.c_uint64),
                                                  ctypes.POINTER(ctypes.c_uint64)]
            L.fp8bq_debug_take_bounds.restype = i32
            _lib = L
    return _lib


def _ptr(a) -> int:
    """Pointer value of an int, None, or a tensor-like with data_ptr()."""
    if a is None:
        return 0
    if isinstance(a, int):
        return a
    return int(a.data_ptr())


def _stream(stream) -> int:
    if stream is None:
        import torch
        if not torch.cuda.is_available():
            return 0  # no device: the library reports FP8BQ_ERR_DEVICE itself
        return int(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return stream
    return int(stream.cuda_stream)


# ----------------------------------------------------------------- C entry points


def fp8bq_quantize(x, dtype_in: int, M: int, N: int, ld: int, block_m: int, block_n: int,
                   y_u8, descale_f32, stream=None) -> int:
    """``fp8bq_quantize`` of the C ABI; pointers may be ints or tensors.
    Returns the fp8bq_status code."""
    return lib().fp8bq_quantize(_ptr(x), dtype_in, M, N, ld, block_m, block_n, _ptr(y_u8),
                                _ptr(descale_f32), _stream(stream))


def fp8bq_quantize_batched(desc_table: Sequence[fp8bq_desc] | ctypes.Array, n_tensors=None,
                           stream=None) -> int:
    """``fp8bq_quantize_batched`` of the C ABI.  Returns the status code."""
    if not isinstance(desc_table, ctypes.Array):
        desc_table = (fp8bq_desc * len(desc_table))(*desc_table)
    n = len(desc_table) if n_tensors is None else n_tensors
    return lib().fp8bq_quantize_batched(desc_table, n, _stream(stream))


def fp8bq_dequantize(y_u8, descale_f32, batch: int, M: int, N: int, block_m: int, block_n: int,
                     out, dtype_out: int, ld_out: int, out_batch_stride: int, stream=None) -> int:
    """``fp8bq_dequantize`` of the C ABI.  Returns the status code."""
    return lib().fp8bq_dequantize(_ptr(y_u8), _ptr(descale_f32), batch, M, N, block_m, block_n,
                                  _ptr(out), dtype_out, ld_out, out_batch_stride,
                                  _stream(stream))


def fp8bq_dequantize_batched(desc_table, n_tensors=None, stream=None) -> int:
    """``fp8bq_dequantize_batched`` of the C ABI.  Returns the status code."""
    if not isinstance(desc_table, ctypes.Array):
        desc_table = (fp8bq_dequant_desc * len(desc_table))(*desc_table)
    n = len(desc_table) if n_tensors is None else n_tensors
    return lib().fp8bq_dequantize_batched(desc_table, n, _stream(stream))


def fp8bq_tensor_scale(desc_table, scale_out, n_tensors=None, stream=None) -> int:
    """``fp8bq_tensor_scale`` of the C ABI.  Returns the status code."""
    if not isinstance(desc_table, ctypes.Array):
        desc_table = (fp8bq_scale_desc * len(desc_table))(*desc_table)
    n = len(desc_table) if n_tensors is None else n_tensors
    return lib().fp8bq_tensor_scale(desc_table, n, _ptr(scale_out), _stream(stream))


def fp8bq_status_string(status: int) -> str:
    return lib().fp8bq_status_string(status).decode()


def fp8bq_sync_status(stream=None) -> int:
    return lib().fp8bq_sync_status(_stream(stream))


def fp8bq_version() -> int:
    return lib().fp8bq_version()


def fp8bq_set_path(path: int) -> int:
    return lib().fp8bq_set_path(path)


def fp8bq_get_path() -> int:
    return lib().fp8bq_get_path()


def fp8bq_set_pdl(enable: int) -> int:
    return lib().fp8bq_set_pdl(int(enable))


def fp8bq_get_pdl() -> int:
    return lib().fp8bq_get_pdl()


def fp8bq_path_for(desc: fp8bq_desc) -> int:
    return lib().fp8bq_path_for(ctypes.byref(desc))


def fp8bq_launch_count(desc_table, n_tensors=None) -> int:
    """``fp8bq_launch_count`` of the C ABI: kernel launches the grouped call
    would enqueue (-1 if it would fail)."""
    if not isinstance(desc_table, ctypes.Array):
        desc_table = (fp8bq_desc * len(desc_table))(*desc_table)
    n = len(desc_table) if n_tensors is None else n_tensors
    return lib().fp8bq_launch_count(desc_table, n)


def fp8bq_debug_set_wait_limit_ns(ns: int) -> int:
    return lib().fp8bq_debug_set_wait_limit_ns(ns)


def fp8bq_debug_set_inject(flags: int) -> int:
    return lib().fp8bq_debug_set_inject(flags)


def fp8bq_checked_build() -> int:
    return lib().fp8bq_checked_build()


def fp8bq_debug_take_bounds() -> tuple[int, int, int]:
    """``fp8bq_debug_take_bounds``: (status, count, first_address)."""
    c, f = ctypes.c_uint64(0), ctypes.c_uint64(0)
    st = lib().fp8bq_debug_take_bounds(ctypes.byref(c), ctypes.byref(f))
    return st, int(c.value), int(f.value)


def check(status: int, what: str = "") -> None:
    if status != FP8BQ_OK:
        raise Fp8bqError(status, what)


# ----------------------------------------------------------------- PyTorch conveniences


def _check_cuda(t, what: str) -> None:
    """The library reads and writes device memory of the current device: refuse
    anything else here, before a kernel could touch a host address."""
    import torch
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{what} must be a CUDA tensor")
    cur = torch.cuda.current_device()
    if t.device.index != cur:
        raise ValueError(f"{what} is on {t.device}, not on the current device cuda:{cur}")


def _dtype_code(t) -> int:
    import torch
    if t.dtype == torch.bfloat16:
        return FP8BQ_BF16
    if t.dtype == torch.float32:
        return FP8BQ_F32
    raise TypeError(f"input must be bfloat16 or float32, got {t.dtype}")


def make_desc(x, y, s, block=DEFAULT_BLOCK) -> fp8bq_desc:
    """Descriptor for a CUDA tensor ``x`` of shape [M, N] or [E, M, N] (unit
    stride along N), its e4m3fn output ``y`` (contiguous, same shape) and its
    descale ``s`` (contiguous [(E,) ceil(M/bm), ceil(N/bn)])."""
    if x.dim() not in (2, 3):
        raise ValueError("expected a 2-D weight or a 3-D stack of expert weights")
    _check_cuda(x, "the input")
    _check_cuda(y, "the e4m3fn output")
    _check_cuda(s, "the descale output")
    if x.shape[-1] > 1 and x.stride(-1) != 1:
        raise ValueError("the last dimension of the input must have unit stride")
    d = fp8bq_desc()
    d.x, d.y_u8, d.descale_f32 = _ptr(x), _ptr(y), _ptr(s)
    d.M, d.N = int(x.shape[-2]), int(x.shape[-1])
    d.ld = int(x.stride(-2)) if x.shape[-2] > 1 else max(int(x.shape[-1]), 1)
    d.ld = max(d.ld, d.N)
    d.batch = int(x.shape[0]) if x.dim() == 3 else 1
    gm, gn = -(-d.M // block[0]), -(-d.N // block[1])
    d.x_batch_stride = int(x.stride(0)) if x.dim() == 3 else 0
    d.y_batch_stride = d.M * d.N if x.dim() == 3 else 0
    d.s_batch_stride = gm * gn if x.dim() == 3 else 0
    d.dtype_in = _dtype_code(x)
    d.block_m, d.block_n = int(block[0]), int(block[1])
    return d


def _on_stream(stream):
    """Context in which PyTorch allocates for ``stream``: outputs the library
    writes on a stream other than the current one are allocated on that
    stream, so the caching allocator cannot hand their memory to another
    stream's work while the kernel still writes it."""
    import contextlib

    import torch
    if stream is None:
        return contextlib.nullcontext()
    if isinstance(stream, int):
        stream = torch.cuda.ExternalStream(stream)
    return torch.cuda.stream(stream)


def _outputs(x, block):
    import torch
    M, N = x.shape[-2], x.shape[-1]
    gm, gn = -(-M // block[0]), -(-N // block[1])
    y = torch.empty(x.shape, dtype=torch.float8_e4m3fn, device=x.device)
    s = torch.empty((*x.shape[:-2], gm, gn), dtype=torch.float32, device=x.device)
    return y, s


def scaled_fp8_blockwise(data_hp, weight_block_size=DEFAULT_BLOCK, stream=None):
    """Quantize one bf16/fp32 CUDA weight ([M, N], or [E, M, N] for a stack of
    experts) to e4m3fn with one fp32 descale per block.

    Returns ``(fp8_data, descale)``: ``fp8_data`` has the input's shape and
    dtype ``torch.float8_e4m3fn``; ``descale`` is [(E,) ceil(M/bm), ceil(N/bn)]
    fp32 (the "weight_scale_inv" of the rollout engine).
    """
    block = tuple(int(b) for b in weight_block_size)
    _check_cuda(data_hp, "data_hp")
    with _on_stream(stream):
        y, s = _outputs(data_hp, block)
    if data_hp.dim() == 2 and (data_hp.shape[-1] <= 1 or data_hp.stride(-1) == 1):
        M, N = data_hp.shape
        ld = max(data_hp.stride(0) if M > 1 else max(N, 1), N)
        st = lib().fp8bq_quantize(data_hp.data_ptr(), _dtype_code(data_hp), M, N, ld, block[0],
                                  block[1], y.data_ptr(), s.data_ptr(), _stream(stream))
    else:
        st = fp8bq_quantize_batched([make_desc(data_hp, y, s, block)], stream=stream)
    check(st, "scaled_fp8_blockwise")
    return y, s


def dequantize_fp8_blockwise(fp8_data, descale, weight_block_size=DEFAULT_BLOCK,
                             out_dtype=None, stream=None):
    """Reverse map of ``scaled_fp8_blockwise``: decode(fp8_data) * descale per
    block, as bf16 (default) or fp32, same shape as ``fp8_data``."""
    import torch
    out_dtype = torch.bfloat16 if out_dtype is None else out_dtype
    if out_dtype not in (torch.bfloat16, torch.float32):
        raise TypeError("out_dtype must be torch.bfloat16 or torch.float32")
    _check_cuda(fp8_data, "fp8_data")
    _check_cuda(descale, "descale")
    if not fp8_data.is_contiguous() or not descale.is_contiguous():
        raise ValueError("fp8_data and descale must be contiguous")
    bm, bn = (int(b) for b in weight_block_size)
    M, N = fp8_data.shape[-2], fp8_data.shape[-1]
    batch = fp8_data.shape[0] if fp8_data.dim() == 3 else 1
    with _on_stream(stream):
        out = torch.empty(fp8_data.shape, dtype=out_dtype, device=fp8_data.device)
    check(fp8bq_dequantize(fp8_data, descale, batch, M, N, bm, bn, out,
                           FP8BQ_BF16 if out_dtype == torch.bfloat16 else FP8BQ_F32, N, M * N,
                           stream), "dequantize_fp8_blockwise")
    return out


def tensor_scales(tensors, stream=None):
    """Per-tensor FP8 scales max(max|x|, eps) / 448 of contiguous bf16/fp32
    CUDA tensors (e.g. this step's Q, K and V), in one grouped call; returns a
    float32 CUDA tensor of len(tensors) scales."""
    import torch
    tensors = list(tensors)
    if not tensors:
        raise ValueError("no tensors")
    _check_cuda(tensors[0], "every tensor")
    with _on_stream(stream):
        out = torch.empty(len(tensors), dtype=torch.float32, device=tensors[0].device)
    descs = []
    for t in tensors:
        _check_cuda(t, "every tensor")
        if not t.is_contiguous():
            raise ValueError("tensors must be contiguous")
        d = fp8bq_scale_desc()
        d.x, d.numel, d.dtype_in, d.reserved = _ptr(t), t.numel(), _dtype_code(t), 0
        descs.append(d)
    check(fp8bq_tensor_scale(descs, out, stream=stream), "tensor_scales")
    return out


# fp8bq_desc as a numpy record (the same 96-byte layout), so that a whole
# table is built from one list of tuples instead of field by field.
_DESC_RECORD = [("x", "<u8"), ("y_u8", "<u8"), ("descale_f32", "<u8"), ("M", "<i8"),
                ("N", "<i8"), ("ld", "<i8"), ("batch", "<i8"), ("x_batch_stride", "<i8"),
                ("y_batch_stride", "<i8"), ("s_batch_stride", "<i8"), ("dtype_in", "<i4"),
                ("block_m", "<i4"), ("block_n", "<i4"), ("reserved", "<i4")]


def _plan_weights(named, bm: int, bn: int, stream=None):
    """Descriptor table (a numpy record array) and output views of
    quant_weights: the fp8 weights are views of one allocation and the
    descales of another, each piece at a 256-byte aligned offset."""
    import numpy as np
    import torch
    cur = torch.cuda.current_device() if torch.cuda.is_available() else -1
    rows = []
    yo = so = 0
    for name, w in named:
        if not isinstance(w, torch.Tensor) or not w.is_cuda or w.device.index != cur:
            _check_cuda(w, name)  # raises with the reason
        shape = w.shape
        if len(shape) not in (2, 3):
            raise ValueError(f"{name}: expected a 2-D weight or a 3-D stack of expert weights")
        M, N = shape[-2], shape[-1]
        if N > 1 and w.stride(-1) != 1:
            raise ValueError(f"{name}: the last dimension of the input must have unit stride")
        dt = FP8BQ_BF16 if w.dtype == torch.bfloat16 else _dtype_code(w)
        gm, gn = -(-M // bm), -(-N // bn)
        stack = len(shape) == 3
        E = shape[0] if stack else 1
        rows.append((w, shape, yo, so, gm, gn, E, M, N, stack, dt))
        yo += (E * M * N + 255) & ~255
        so += (E * gm * gn + 63) & ~63
    dev = named[0][1].device
    with _on_stream(stream):
        ybuf = torch.empty(max(yo, 1), dtype=torch.uint8, device=dev).view(torch.float8_e4m3fn)
        sbuf = torch.empty(max(so, 1), dtype=torch.float32, device=dev)
    yp, sp = ybuf.data_ptr(), sbuf.data_ptr()
    recs, outs = [], []
    for (name, _w), (w, shape, yoff, soff, gm, gn, E, M, N, stack, dt) in zip(named, rows):
        ld = max(w.stride(-2) if M > 1 else max(N, 1), N)
        recs.append((w.data_ptr(), yp + yoff, sp + 4 * soff, M, N, ld, E,
                     w.stride(0) if stack else 0, M * N if stack else 0,
                     gm * gn if stack else 0, dt, bm, bn, 0))
        if stack:
            y = ybuf.as_strided((E, M, N), (M * N, N, 1), yoff)
            s = sbuf.as_strided((E, gm, gn), (gm * gn, gn, 1), soff)
        else:
            y = ybuf.as_strided((M, N), (N, 1), yoff)
            s = sbuf.as_strided((gm, gn), (gn, 1), soff)
        outs.append((name, y))
        outs.append((name + "_scale_inv", s))
    return np.array(recs, dtype=_DESC_RECORD), outs


def quant_weights(weights: Iterable, weight_block_size=DEFAULT_BLOCK, stream=None):
    """Quantize every (name, tensor) pair in one grouped call and return the
    list the rollout engine loads: (name, fp8 weight) followed by
    (name + "_scale_inv", descale) for each input, in input order.

    The fp8 weights are views of one device allocation and the descales of
    another (each piece at a 256-byte aligned offset), so a whole model costs
    two allocations; the memory is returned when the last view is freed."""
    bm, bn = (int(b) for b in weight_block_size)
    named = list(weights)
    if not named:
        return []
    table, out = _plan_weights(named, bm, bn, stream)
    st = lib().fp8bq_quantize_batched(table.ctypes.data_as(ctypes.POINTER(fp8bq_desc)),
                                      len(named), _stream(stream))
    check(st, "quant_weights")
    return out
