"""Host-side tests of the C ABI: the library loads, exports every entry point
the header declares, and rejects bad arguments before touching a device.

These run without a GPU: argument checks happen before any CUDA call, and a
valid call with no usable device returns FP8BQ_ERR_DEVICE.
"""
import ctypes
import os
import re

import pytest
import torch

import blockwise_fp8_weight_b200 as fq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fp8bq.h")
NO_GPU = not torch.cuda.is_available()

# fake, well-aligned device addresses: never dereferenced by the host checks
X, Y, S = 0x7000_0000_0000, 0x7100_0000_0000, 0x7200_0000_0000


def declared_functions():
    text = open(HEADER).read()
    return re.findall(r"FP8BQ_API\s+[\w\s\*]+?\b(fp8bq_\w+)\s*\(", text)


def test_header_declares_the_entry_points():
    names = declared_functions()
    for must in ("fp8bq_quantize", "fp8bq_quantize_batched", "fp8bq_status_string",
                 "fp8bq_sync_status"):
        assert must in names


def test_library_exports_every_declared_symbol():
    L = fq.lib()
    for name in declared_functions():
        assert hasattr(L, name), name
        assert callable(getattr(L, name))


def test_version_and_struct_layout():
    assert fq.fp8bq_version() == 10000
    assert ctypes.sizeof(fq.fp8bq_desc) == 96
    assert fq.fp8bq_desc.dtype_in.offset == 80
    assert fq.fp8bq_desc.block_n.offset == 88


@pytest.mark.parametrize("M,N,block,path", [
    (1, 1 << 22, (128, 128), fq.FP8BQ_PATH_VECTOR),  # 8 MB, one row: 1-row blocks, folded
    (1, 1024, (128, 128), fq.FP8BQ_PATH_TMA),        # 2 KB: below the size, planned as given
    (8, 1 << 20, (128, 128), fq.FP8BQ_PATH_VECTOR),  # blocks of its 8 rows
    (40, 1 << 18, (128, 128), fq.FP8BQ_PATH_TMA),    # more than a quarter block: as given
    (1, 1 << 22, (1, 128), fq.FP8BQ_PATH_VECTOR),
])
def test_few_row_planning_without_a_device(M, N, block, path):
    """fp8bq_path_for reports the variant of the planner's equivalent geometry
    for few-row tensors of at least 4 MiB (host only, no device needed)."""
    d = fq.fp8bq_desc()
    d.x, d.y_u8, d.descale_f32 = X, Y, S
    d.M, d.N, d.ld, d.batch = M, N, N, 1
    d.dtype_in, (d.block_m, d.block_n) = fq.FP8BQ_BF16, block
    assert fq.fp8bq_path_for(d) == path


def test_numpy_descriptor_record_matches_the_struct():
    """quant_weights builds its descriptor table as a numpy record array: the
    same size and field offsets as struct fp8bq_desc."""
    import numpy as np
    rec = np.dtype(fq._DESC_RECORD)
    assert rec.itemsize == ctypes.sizeof(fq.fp8bq_desc)
    assert [n for n, _ in fq._DESC_RECORD] == [n for n, _ in fq.fp8bq_desc._fields_]
    for name, _ in fq._DESC_RECORD:
        assert rec.fields[name][1] == getattr(fq.fp8bq_desc, name).offset, name


def test_status_strings():
    for code in range(12):
        s = fq.fp8bq_status_string(code)
        assert s.startswith("FP8BQ_")
    assert "unknown" in fq.fp8bq_status_string(1234)


def q(**kw):
    a = dict(x=X, dtype_in=fq.FP8BQ_BF16, M=256, N=384, ld=384, block_m=128, block_n=128,
             y_u8=Y, descale_f32=S, stream=0)
    a.update(kw)
    return fq.fp8bq_quantize(**a)


@pytest.mark.parametrize("kw,status", [
    (dict(dtype_in=2), fq.FP8BQ_ERR_DTYPE),
    (dict(dtype_in=-1), fq.FP8BQ_ERR_DTYPE),
    (dict(block_m=0), fq.FP8BQ_ERR_BLOCK),
    (dict(block_n=-3), fq.FP8BQ_ERR_BLOCK),
    (dict(block_m=256, block_n=257), fq.FP8BQ_ERR_BLOCK),
    (dict(M=-1), fq.FP8BQ_ERR_SHAPE),
    (dict(N=-1, ld=0), fq.FP8BQ_ERR_SHAPE),
    (dict(ld=383), fq.FP8BQ_ERR_SHAPE),
    (dict(M=1 << 31, N=1, ld=1), fq.FP8BQ_ERR_SHAPE),
    (dict(M=1 << 30, N=4, ld=1 << 40), fq.FP8BQ_ERR_SHAPE),   # byte offsets beyond 2^62
    (dict(x=0), fq.FP8BQ_ERR_NULL),
    (dict(y_u8=0), fq.FP8BQ_ERR_NULL),
    (dict(descale_f32=0), fq.FP8BQ_ERR_NULL),
    (dict(x=X + 1), fq.FP8BQ_ERR_ALIGN),
    (dict(dtype_in=fq.FP8BQ_F32, x=X + 2), fq.FP8BQ_ERR_ALIGN),
    (dict(descale_f32=S + 2), fq.FP8BQ_ERR_ALIGN),
    (dict(y_u8=X + 1000), fq.FP8BQ_ERR_OVERLAP),          # y inside x
    (dict(descale_f32=Y + 256 * 384 - 4), fq.FP8BQ_ERR_OVERLAP),  # s overlaps y's tail
    (dict(x=Y - 2 * 384 + 2), fq.FP8BQ_ERR_OVERLAP),      # x runs into y
])
def test_argument_errors(kw, status):
    assert q(**kw) == status


def test_empty_tensors_are_a_no_op():
    assert q(M=0, x=0, y_u8=0, descale_f32=0) == fq.FP8BQ_OK
    assert q(N=0, ld=0) == fq.FP8BQ_OK
    assert fq.fp8bq_quantize_batched([]) == fq.FP8BQ_OK


@pytest.mark.skipif(not NO_GPU, reason="checks the no-device path")
def test_valid_call_without_device_reports_device_error():
    assert q() == fq.FP8BQ_ERR_DEVICE
    assert q(x=X + 2) == fq.FP8BQ_ERR_DEVICE   # misaligned-for-vectors is still valid input


def desc(**kw):
    d = fq.fp8bq_desc()
    a = dict(x=X, y_u8=Y, descale_f32=S, M=1536, N=2048, ld=2048, batch=128,
             x_batch_stride=1536 * 2048, y_batch_stride=1536 * 2048, s_batch_stride=12 * 16,
             dtype_in=fq.FP8BQ_BF16, block_m=128, block_n=128, reserved=0)
    a.update(kw)
    for k, v in a.items():
        setattr(d, k, v)
    return d


def test_batched_argument_errors():
    assert fq.fp8bq_quantize_batched([desc()], n_tensors=-1) == fq.FP8BQ_ERR_ARG
    assert fq.fp8bq_quantize_batched([desc(batch=-1)]) == fq.FP8BQ_ERR_SHAPE
    assert fq.fp8bq_quantize_batched([desc(x_batch_stride=-5)]) == fq.FP8BQ_ERR_SHAPE
    # experts' outputs would overlap each other
    assert fq.fp8bq_quantize_batched([desc(y_batch_stride=1536 * 2048 - 1)]) == fq.FP8BQ_ERR_OVERLAP
    assert fq.fp8bq_quantize_batched([desc(s_batch_stride=191)]) == fq.FP8BQ_ERR_OVERLAP
    # two tensors writing the same output
    a = desc()
    b = desc(x=X + (1 << 36))
    assert fq.fp8bq_quantize_batched([a, b]) == fq.FP8BQ_ERR_OVERLAP
    # second tensor reads the first one's descale
    b = desc(x=S, batch=1, M=4, N=8, ld=8, y_u8=Y + (1 << 36), descale_f32=S + (1 << 36))
    assert fq.fp8bq_quantize_batched([a, b]) == fq.FP8BQ_ERR_OVERLAP
    # one bad descriptor anywhere rejects the whole list
    c = desc(x=X + (1 << 38), y_u8=Y + (1 << 38), descale_f32=S + (1 << 38), block_m=0)
    assert fq.fp8bq_quantize_batched([a, c]) == fq.FP8BQ_ERR_BLOCK


@pytest.mark.skipif(not NO_GPU, reason="the fake pointers must never reach a launch")
def test_inputs_may_overlap_each_other():
    a = desc(batch=1)
    b = desc(batch=1, y_u8=Y + (1 << 36), descale_f32=S + (1 << 36))   # same input
    # passes every argument check; only the missing device stops it
    assert fq.fp8bq_quantize_batched([a, b]) == fq.FP8BQ_ERR_DEVICE


@pytest.fixture
def path_guard():
    yield
    fq.fp8bq_set_path(fq.FP8BQ_PATH_AUTO)


def test_launch_count_refuses_what_the_call_refuses():
    assert fq.fp8bq_launch_count([desc(block_m=0)]) == -1        # invalid block
    assert fq.fp8bq_launch_count([desc()], n_tensors=-1) == -1   # negative count
    # a valid call needs a usable device to be planned (none in this container
    # means -1; on a B200 the GPU tests check the counts)
    if not torch.cuda.is_available():
        assert fq.fp8bq_launch_count([desc()]) == -1


def test_variant_choice(path_guard):
    P = fq.fp8bq_path_for
    assert fq.fp8bq_get_path() == fq.FP8BQ_PATH_AUTO
    assert P(desc()) == fq.FP8BQ_PATH_TMA                          # 128x128, aligned
    assert P(desc(batch=1, block_m=1, block_n=128)) == fq.FP8BQ_PATH_VECTOR  # small blocks
    assert P(desc(batch=1, block_m=64, block_n=64)) == fq.FP8BQ_PATH_VECTOR
    assert P(desc(batch=1, block_m=32, block_n=16)) == fq.FP8BQ_PATH_VECTOR  # no TMA geometry
    assert P(desc(batch=1, block_m=1, block_n=16)) == fq.FP8BQ_PATH_VECTOR   # 8 KB slots
    assert P(desc(dtype_in=fq.FP8BQ_F32)) == fq.FP8BQ_PATH_TMA
    assert fq.fp8bq_set_path(fq.FP8BQ_PATH_VECTOR) == fq.FP8BQ_OK
    assert P(desc()) == fq.FP8BQ_PATH_VECTOR
    assert fq.fp8bq_set_path(fq.FP8BQ_PATH_AUTO) == fq.FP8BQ_OK
    # rows only 8-byte aligned: the vector kernel in 8-byte halves
    assert P(desc(batch=1, N=4100, ld=4100)) == fq.FP8BQ_PATH_VECTOR
    assert P(desc(batch=1, N=4096, ld=4100)) == fq.FP8BQ_PATH_VECTOR
    assert P(desc(x=X + 8)) == fq.FP8BQ_PATH_VECTOR
    assert P(desc(y_u8=Y + 4)) == fq.FP8BQ_PATH_VECTOR
    assert P(desc(batch=1, N=4100, ld=4100, dtype_in=fq.FP8BQ_F32)) == fq.FP8BQ_PATH_TMA
    assert P(desc(batch=1, N=4098, ld=4098, dtype_in=fq.FP8BQ_F32)) == fq.FP8BQ_PATH_VECTOR
    # narrower than that: the generic kernel
    assert P(desc(batch=1, N=4102, ld=4102)) == fq.FP8BQ_PATH_GENERIC   # rows 4-byte aligned
    assert P(desc(batch=1, N=4097, ld=4100)) == fq.FP8BQ_PATH_GENERIC   # codes rows odd
    assert P(desc(batch=1, N=4097, ld=4097, dtype_in=fq.FP8BQ_F32)) == fq.FP8BQ_PATH_GENERIC
    assert P(desc(x=X + 2)) == fq.FP8BQ_PATH_GENERIC
    assert P(desc(x=X + 4)) == fq.FP8BQ_PATH_GENERIC
    assert P(desc(y_u8=Y + 2)) == fq.FP8BQ_PATH_GENERIC
    assert P(desc(x_batch_stride=1536 * 2048 + 2)) == fq.FP8BQ_PATH_GENERIC
    assert P(desc(batch=1, block_m=5, block_n=7)) == fq.FP8BQ_PATH_GENERIC
    assert P(desc(batch=1, block_m=256, block_n=256)) == fq.FP8BQ_PATH_GENERIC  # 65536 elements
    assert P(desc(block_m=0)) == -1
    assert fq.fp8bq_set_path(fq.FP8BQ_PATH_TMA) == fq.FP8BQ_OK
    assert P(desc()) == fq.FP8BQ_PATH_TMA
    assert P(desc(dtype_in=fq.FP8BQ_F32)) == fq.FP8BQ_PATH_TMA
    assert P(desc(batch=1, block_m=1, block_n=128)) == fq.FP8BQ_PATH_TMA    # stacked blocks
    assert P(desc(batch=1, block_m=64, block_n=64)) == fq.FP8BQ_PATH_TMA
    assert P(desc(batch=1, N=4100, ld=4100)) == fq.FP8BQ_PATH_VECTOR   # no tensor map
    assert P(desc(batch=1, N=4102, ld=4102)) == fq.FP8BQ_PATH_GENERIC
    assert fq.fp8bq_set_path(fq.FP8BQ_PATH_GENERIC) == fq.FP8BQ_OK
    assert P(desc()) == fq.FP8BQ_PATH_GENERIC
    assert fq.fp8bq_set_path(7) == fq.FP8BQ_ERR_ARG
    assert fq.fp8bq_get_path() == fq.FP8BQ_PATH_GENERIC


def test_pdl_switch():
    assert fq.fp8bq_get_pdl() == 1                       # on by default
    try:
        assert fq.fp8bq_set_pdl(0) == fq.FP8BQ_OK
        assert fq.fp8bq_get_pdl() == 0
        assert fq.fp8bq_set_pdl(5) == fq.FP8BQ_OK
        assert fq.fp8bq_get_pdl() == 1
    finally:
        fq.fp8bq_set_pdl(1)


def test_debug_knobs():
    assert fq.fp8bq_debug_set_inject(2) == fq.FP8BQ_ERR_ARG
    assert fq.fp8bq_debug_set_inject(0) == fq.FP8BQ_OK
    assert fq.fp8bq_debug_set_wait_limit_ns(0) == fq.FP8BQ_OK


@pytest.mark.skipif(not NO_GPU, reason="checks the no-device path")
def test_sync_status_without_device():
    assert fq.fp8bq_sync_status(0) == fq.FP8BQ_ERR_DEVICE


def dq(**kw):
    a = dict(y_u8=Y, descale_f32=S, batch=1, M=256, N=384, block_m=128, block_n=128, out=X,
             dtype_out=fq.FP8BQ_BF16, ld_out=384, out_batch_stride=0, stream=0)
    a.update(kw)
    return fq.fp8bq_dequantize(**a)


@pytest.mark.parametrize("kw,status", [
    (dict(dtype_out=3), fq.FP8BQ_ERR_DTYPE),
    (dict(block_m=0), fq.FP8BQ_ERR_BLOCK),
    (dict(block_m=512, block_n=512), fq.FP8BQ_ERR_BLOCK),
    (dict(M=-2), fq.FP8BQ_ERR_SHAPE),
    (dict(ld_out=100), fq.FP8BQ_ERR_SHAPE),
    (dict(batch=-1), fq.FP8BQ_ERR_SHAPE),
    (dict(batch=2, out_batch_stride=-1), fq.FP8BQ_ERR_SHAPE),
    (dict(batch=2, out_batch_stride=256 * 384 - 1), fq.FP8BQ_ERR_OVERLAP),
    (dict(y_u8=0), fq.FP8BQ_ERR_NULL),
    (dict(out=0), fq.FP8BQ_ERR_NULL),
    (dict(out=X + 1), fq.FP8BQ_ERR_ALIGN),
    (dict(dtype_out=fq.FP8BQ_F32, out=X + 2), fq.FP8BQ_ERR_ALIGN),
    (dict(descale_f32=S + 1), fq.FP8BQ_ERR_ALIGN),
    (dict(out=Y - 100), fq.FP8BQ_ERR_OVERLAP),
    (dict(out=S), fq.FP8BQ_ERR_OVERLAP),
])
def test_dequantize_argument_errors(kw, status):
    assert dq(**kw) == status


def test_dequantize_empty_and_no_device():
    assert dq(M=0, y_u8=0, out=0, descale_f32=0) == fq.FP8BQ_OK
    assert dq(batch=0) == fq.FP8BQ_OK
    if NO_GPU:
        assert dq() == fq.FP8BQ_ERR_DEVICE


def ddesc(**kw):
    d = fq.fp8bq_dequant_desc()
    a = dict(y_u8=Y, descale_f32=S, out=X, batch=1, M=256, N=384, ld_out=384, out_batch_stride=0,
             dtype_out=fq.FP8BQ_BF16, block_m=128, block_n=128, reserved=0)
    a.update(kw)
    for k, v in a.items():
        setattr(d, k, v)
    return d


def test_dequantize_batched_layout_and_errors():
    assert ctypes.sizeof(fq.fp8bq_dequant_desc) == 80
    B = fq.fp8bq_dequantize_batched
    assert B([]) == fq.FP8BQ_OK
    assert B([ddesc()], n_tensors=-1) == fq.FP8BQ_ERR_ARG
    assert B([ddesc(), ddesc(dtype_out=7, out=X + (1 << 36))]) == fq.FP8BQ_ERR_DTYPE
    # two descriptors writing the same output
    assert B([ddesc(), ddesc(y_u8=Y + (1 << 36), descale_f32=S + (1 << 36))]) == \
        fq.FP8BQ_ERR_OVERLAP
    # second descriptor's output runs over the first one's codes
    assert B([ddesc(), ddesc(out=Y, y_u8=Y + (1 << 36), descale_f32=S + (1 << 36))]) == \
        fq.FP8BQ_ERR_OVERLAP
    if NO_GPU:
        assert B([ddesc(), ddesc(out=X + (1 << 36))]) == fq.FP8BQ_ERR_DEVICE


def sdesc(**kw):
    d = fq.fp8bq_scale_desc()
    a = dict(x=X, numel=4096, dtype_in=fq.FP8BQ_BF16, reserved=0)
    a.update(kw)
    for k, v in a.items():
        setattr(d, k, v)
    return d


def test_tensor_scale_argument_errors():
    T = lambda descs, out=S, n=None: fq.fp8bq_tensor_scale(descs, out, n_tensors=n)  # noqa: E731
    assert ctypes.sizeof(fq.fp8bq_scale_desc) == 24
    assert T([sdesc()], n=-1) == fq.FP8BQ_ERR_ARG
    assert T([], n=0) == fq.FP8BQ_OK
    assert T([sdesc()], out=0) == fq.FP8BQ_ERR_NULL
    assert T([sdesc()], out=S + 2) == fq.FP8BQ_ERR_ALIGN
    assert T([sdesc(dtype_in=5)]) == fq.FP8BQ_ERR_DTYPE
    assert T([sdesc(numel=-1)]) == fq.FP8BQ_ERR_SHAPE
    assert T([sdesc(x=0)]) == fq.FP8BQ_ERR_NULL
    assert T([sdesc(x=X + 1)]) == fq.FP8BQ_ERR_ALIGN
    assert T([sdesc(x=S - 100)]) == fq.FP8BQ_ERR_OVERLAP
    if NO_GPU:
        assert T([sdesc(), sdesc(x=0, numel=0)]) == fq.FP8BQ_ERR_DEVICE


def test_conveniences_refuse_host_tensors():
    """The PyTorch conveniences hand only device memory of the current device
    to the library: host tensors are refused before any call into it."""
    import torch
    w = torch.zeros(256, 384, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA tensor"):
        fq.scaled_fp8_blockwise(w)
    with pytest.raises(ValueError, match="CUDA tensor"):
        fq.quant_weights([("layers.0.q_proj.weight", w)])
    with pytest.raises(ValueError, match="CUDA tensor"):
        fq.tensor_scales([w])
    y = torch.zeros(256, 384, dtype=torch.uint8)
    s = torch.zeros(2, 3, dtype=torch.float32)
    with pytest.raises(ValueError, match="CUDA tensor"):
        fq.dequantize_fp8_blockwise(y, s)
    with pytest.raises(ValueError, match="CUDA tensor"):
        fq.make_desc(w, y, s)


def test_c_consumer_compiles_links_and_runs(tmp_path):
    """tests/c/abi_consumer.c: the header is C99, every declared entry point
    links from plain C, the descriptor sizes are the documented ones, and the
    device-free calls behave as documented."""
    import shutil
    import subprocess
    from blockwise_fp8_weight_b200 import build as B
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    fq.lib()  # builds the library if needed
    cuda_inc = os.path.join(os.path.dirname(os.path.dirname(os.path.realpath(B.nvcc()))), "include")
    exe = str(tmp_path / "abi_consumer")
    pkg = os.path.dirname(fq.LIB_PATH)
    subprocess.run([gcc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
                    "-I", cuda_inc, os.path.join(ROOT, "tests", "c", "abi_consumer.c"), "-L", pkg,
                    "-lfp8bq", f"-Wl,-rpath,{pkg}", "-o", exe], check=True)
    r = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stderr
    assert "abi consumer ok" in r.stdout
