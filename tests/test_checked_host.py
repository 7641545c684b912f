"""Host-side tests of the bounds-checked build (libfp8bq_checked.so, compiled
with FP8BQ_CHECKED=1): it loads, exports every entry point the header
declares, says that it is the checked build, accepts the output-trimming
knob that the default build refuses, and rejects bad arguments exactly as the
default build does.  No GPU is needed."""
import ctypes
import re

import pytest
import torch

import blockwise_fp8_weight_b200 as fq
from blockwise_fp8_weight_b200 import build as cuda_build
from tests.test_abi_host import HEADER, X, Y, S

NO_GPU = not torch.cuda.is_available()


def declared_functions():
    return re.findall(r"FP8BQ_API\s+[\w\s\*]+?\b(fp8bq_\w+)\s*\(", open(HEADER).read())


@pytest.fixture(scope="module")
def checked():
    L = ctypes.CDLL(cuda_build.build(checked=True))
    L.fp8bq_debug_take_bounds.argtypes = [ctypes.POINTER(ctypes.c_uint64)] * 2
    L.fp8bq_debug_set_inject.argtypes = [ctypes.c_uint32]
    L.fp8bq_status_string.restype = ctypes.c_char_p
    L.fp8bq_quantize.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_int64,
                                 ctypes.c_int64, ctypes.c_int, ctypes.c_int, ctypes.c_void_p,
                                 ctypes.c_void_p, ctypes.c_void_p]
    yield L
    L.fp8bq_debug_set_inject(0)


def test_checked_library_exports_every_declared_symbol(checked):
    for name in declared_functions():
        assert callable(getattr(checked, name)), name


def test_each_build_says_which_it_is(checked):
    assert checked.fp8bq_checked_build() == 1
    assert fq.lib().fp8bq_checked_build() == (1 if fq.CHECKED else 0)


def test_trim_knob_only_in_the_checked_build(checked):
    trim = fq.FP8BQ_INJECT_TRIM_OUTPUTS
    assert checked.fp8bq_debug_set_inject(trim) == fq.FP8BQ_OK
    assert checked.fp8bq_debug_set_inject(trim | fq.FP8BQ_INJECT_DROP_FIRST_LOAD) == fq.FP8BQ_OK
    assert checked.fp8bq_debug_set_inject(4) == fq.FP8BQ_ERR_ARG
    assert checked.fp8bq_debug_set_inject(0) == fq.FP8BQ_OK
    if not fq.CHECKED:
        assert fq.fp8bq_debug_set_inject(trim) == fq.FP8BQ_ERR_ARG
        assert fq.fp8bq_debug_set_inject(0) == fq.FP8BQ_OK


def test_bounds_record_of_the_default_build_is_empty_without_a_device():
    if fq.CHECKED:
        pytest.skip("this process loaded the checked library")
    assert fq.fp8bq_debug_take_bounds() == (fq.FP8BQ_OK, 0, 0)
    assert fq.lib().fp8bq_debug_take_bounds(None, None) == fq.FP8BQ_OK


@pytest.mark.skipif(not NO_GPU, reason="checks the no-device answer")
def test_checked_bounds_record_needs_a_device(checked):
    c, f = ctypes.c_uint64(7), ctypes.c_uint64(7)
    assert checked.fp8bq_debug_take_bounds(ctypes.byref(c), ctypes.byref(f)) == \
        fq.FP8BQ_ERR_DEVICE
    assert (c.value, f.value) == (7, 7)       # untouched on error


def test_bounds_status_string(checked):
    for L in (checked, fq.lib()):
        s = L.fp8bq_status_string(fq.FP8BQ_ERR_DEVICE_BOUNDS)
        assert s.decode().startswith("FP8BQ_ERR_DEVICE_BOUNDS")


@pytest.mark.parametrize("args,status", [
    ((X, 2, 256, 384, 384, 128, 128, Y, S, 0), fq.FP8BQ_ERR_DTYPE),
    ((X, 0, 256, 384, 383, 128, 128, Y, S, 0), fq.FP8BQ_ERR_SHAPE),
    ((X, 0, 256, 384, 384, 0, 128, Y, S, 0), fq.FP8BQ_ERR_BLOCK),
    ((0, 0, 256, 384, 384, 128, 128, Y, S, 0), fq.FP8BQ_ERR_NULL),
    ((X + 1, 0, 256, 384, 384, 128, 128, Y, S, 0), fq.FP8BQ_ERR_ALIGN),
    ((X, 0, 256, 384, 384, 128, 128, X, S, 0), fq.FP8BQ_ERR_OVERLAP),
])
def test_argument_checks_match_the_default_build(checked, args, status):
    assert checked.fp8bq_quantize(*args) == status
    assert fq.fp8bq_quantize(*args[:9], stream=0) == status
