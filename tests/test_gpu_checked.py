"""The bounds-checked build (libfp8bq_checked.so) on the GPU.

  * Its parity: the quantizer, dequantizer, per-tensor-scale and launch-order
    GPU suites run again in a child process that loads the checked library
    (FP8BQ_CHECKED=1).  Every call there ends in fp8bq_sync_status, which in
    a checked build fails on any skipped out-of-range access, so the suites
    prove both that the kernels make no access outside their tensors on those
    cases and that the checks change no output bit.
  * Its checks: with FP8BQ_INJECT_TRIM_OUTPUTS every output is taken as one
    byte shorter than it is, so the last (legitimate) store to each output is
    reported and skipped.  No access outside any buffer is made: the skipped
    stores leave the buffers' fill bytes in place.  (Run by the child process
    above; in a process with the default library these cases skip.)
"""
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

import blockwise_fp8_weight_b200 as fq
import oracle
from blockwise_fp8_weight_b200 import build as cuda_build
from synth import TensorSpec
from synth import workloads as W
from tests.gpu_util import CANARY, Guarded, Outputs, to_device

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SUITES = ["tests/test_gpu_parity.py", "tests/test_gpu_dequant.py", "tests/test_gpu_scale.py",
          "tests/test_gpu_pdl.py", "tests/test_gpu_checked.py"]
checked_only = pytest.mark.skipif(not fq.CHECKED, reason="needs the checked library "
                                  "(run by the child process of the suite test)")


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    yield
    torch.cuda.synchronize()


@pytest.mark.skipif(fq.CHECKED, reason="this process is the checked child")
def test_gpu_suites_under_the_checked_library():
    cuda_build.build(checked=True)
    env = dict(os.environ, FP8BQ_CHECKED="1")
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-m", "gpu",
                        "-p", "no:cacheprovider", *SUITES],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=1800)
    tail = r.stdout[-6000:] + r.stderr[-2000:]
    assert r.returncode == 0, tail
    assert " passed" in r.stdout and " failed" not in r.stdout, tail


@pytest.fixture
def trimmed():
    st, _, _ = fq.fp8bq_debug_take_bounds()            # start from an empty record
    assert st == fq.FP8BQ_OK
    assert fq.fp8bq_debug_set_inject(fq.FP8BQ_INJECT_TRIM_OUTPUTS) == fq.FP8BQ_OK
    yield
    fq.fp8bq_debug_set_inject(0)
    fq.fp8bq_set_path(fq.FP8BQ_PATH_AUTO)
    fq.fp8bq_debug_take_bounds()


def take_record(min_count: int, spans) -> None:
    """The record holds at least min_count skipped accesses, and the address
    it names lies in the last 16 bytes of one of the given (start, size)."""
    assert fq.fp8bq_sync_status() == fq.FP8BQ_ERR_DEVICE_BOUNDS
    st, count, first = fq.fp8bq_debug_take_bounds()
    assert st == fq.FP8BQ_OK and count >= min_count, count
    assert any(p + n - 16 <= first < p + n for p, n in spans), (hex(first), spans)
    assert fq.fp8bq_debug_take_bounds() == (fq.FP8BQ_OK, 0, 0)  # taking clears it


@checked_only
def test_checked_library_is_loaded():
    assert fq.fp8bq_checked_build() == 1


@checked_only
@pytest.mark.parametrize("path,dtype,shape", [
    (fq.FP8BQ_PATH_VECTOR, "bf16", (256, 384)),
    (fq.FP8BQ_PATH_VECTOR, "bf16", (130, 260)),      # rows only 8-byte aligned: halves
    (fq.FP8BQ_PATH_TMA, "bf16", (256, 384)),         # paired TMA tiles
    (fq.FP8BQ_PATH_TMA, "f32", (256, 384)),
    (fq.FP8BQ_PATH_GENERIC, "bf16", (130, 129)),
])
def test_trimmed_quantize_outputs_are_caught_and_skipped(trimmed, path, dtype, shape):
    sp = TensorSpec("trim", *shape, dtype=dtype, seed=31, tensor_id=1)
    x = W.materialize(sp)
    owner, ptr = to_device(x)
    out = Outputs(sp)
    assert fq.fp8bq_set_path(path) == fq.FP8BQ_OK
    assert fq.fp8bq_quantize_batched([out.desc(ptr)]) == fq.FP8BQ_OK
    take_record(2, [(out.y.ptr, out.y.nbytes), (out.s.ptr, out.s.nbytes)])
    assert out.y.canaries_intact() and out.s.canaries_intact()
    yw, sw = oracle.quantize(x, sp.M, sp.N, sp.row_stride, *sp.block)
    y = out.y.numpy()
    s = out.s.numpy()
    want_y = yw.reshape(-1)
    want_s = sw.reshape(-1).view(np.uint8)
    # everything before the last store of each output is the oracle's; the
    # skipped last store left the fill bytes (at most one 8-byte vector of codes)
    assert np.array_equal(y[:-8], want_y[:-8])
    tail = y[-8:]
    assert tail[-1] == CANARY
    assert ((tail == want_y[-8:]) | (tail == CANARY)).all()
    assert np.array_equal(s[:-4], want_s[:-4]) and (s[-4:] == CANARY).all()


@checked_only
@pytest.mark.parametrize("path", [fq.FP8BQ_PATH_VECTOR, fq.FP8BQ_PATH_GENERIC])
def test_trimmed_dequantize_output_is_caught_and_skipped(trimmed, path):
    M, N = 128, 512
    rng = np.random.default_rng(3)
    y = rng.integers(0, 256, size=(M, N), dtype=np.uint8)
    y[(y & 0x7F) == 0x7F] = 0                          # no NaN codes
    s = np.array([[0.5, 2.0, 0.25, 4.0]], dtype=np.float32)
    yt = torch.from_numpy(y.reshape(-1)).cuda()
    st = torch.from_numpy(s.reshape(-1)).cuda()
    out = Guarded(M * N * 2)
    assert fq.fp8bq_set_path(path) == fq.FP8BQ_OK
    assert fq.fp8bq_dequantize(yt, st, 1, M, N, 128, 128, out.ptr, fq.FP8BQ_BF16, N, 0) == \
        fq.FP8BQ_OK
    take_record(1, [(out.ptr, out.nbytes)])
    assert out.canaries_intact()
    got = out.numpy().view(np.uint16)
    want = oracle.dequantize(y, s, 128, 128, "bf16").reshape(-1)
    keep = 8 if path == fq.FP8BQ_PATH_VECTOR else 1    # the skipped store's elements
    assert np.array_equal(got[:-keep], want[:-keep])
    assert (out.numpy()[-2 * keep:] == CANARY).all()


@checked_only
def test_trimmed_tensor_scale_output_is_caught_and_skipped(trimmed):
    xs = [torch.randn(20000, device="cuda").to(torch.bfloat16) for _ in range(3)]
    descs = []
    for x in xs:
        d = fq.fp8bq_scale_desc()
        d.x, d.numel, d.dtype_in, d.reserved = x.data_ptr(), x.numel(), fq.FP8BQ_BF16, 0
        descs.append(d)
    out = Guarded(4 * len(descs))
    assert fq.fp8bq_tensor_scale(descs, out.ptr) == fq.FP8BQ_OK
    take_record(3, [(out.ptr, out.nbytes)])            # zeroing, atomic max, final store
    assert out.canaries_intact()
    got = out.numpy().view(np.float32)
    want = [oracle.tensor_scale(x.float().cpu().numpy()) for x in xs[:2]]
    assert np.array_equal(got[:2].view(np.uint32), np.array(want, np.float32).view(np.uint32))
    assert (out.numpy()[-4:] == CANARY).all()
