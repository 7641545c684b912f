"""GPU parity at the largest sizes the contract allows, where every byte offset
needs 64 bits: single tensors and an expert stack of more than 4 GiB, and a
row at the length limit (N = 2^31 - 128, the largest multiple of the block
below 2^31).  Each is quantized by every kernel family that takes it; sampled
blocks (the corners included, whose offsets lie beyond 4 GiB) are compared
with the oracle block by block, and the families' full outputs with each
other byte for byte.  The widest case is also dequantized and compared with
the oracle's dequantization of the sampled blocks."""
import numpy as np
import pytest
import torch

import blockwise_fp8_weight_b200 as fq
import oracle
from synth import DIST_STUDENT_T3, TensorSpec
from synth import workloads as W
from tests.gpu_util import Guarded, check_sampled, no_nan_codes, run, sample_blocks

pytestmark = pytest.mark.gpu

AUTO, VECTOR, TMA, GENERIC = (fq.FP8BQ_PATH_AUTO, fq.FP8BQ_PATH_VECTOR, fq.FP8BQ_PATH_TMA,
                              fq.FP8BQ_PATH_GENERIC)
CASES = {
    # 2^31.3 elements, 5.4 GB of bf16
    "wide": (TensorSpec("wide", 65536, 40960, seed=71, tensor_id=1, row_lognormal_sigma=0.5),
             [AUTO, VECTOR, GENERIC]),
    # one row of 2^31 - 128 bf16 (4.3 GB), 1 x 128 blocks
    "row_limit": (TensorSpec("row_limit", 1, 2 ** 31 - 128, block=(1, 128), seed=71,
                             tensor_id=2, dist=DIST_STUDENT_T3), [AUTO, TMA, VECTOR]),
    # 160 experts of 2048 x 8192 bf16 (5.4 GB), one descale grid each
    "stack": (TensorSpec("stack", 2048, 8192, batch=160, seed=71, tensor_id=3,
                         batch_lognormal_sigma=0.7), [AUTO, VECTOR]),
    # fp32, 5.4 GB
    "wide_f32": (TensorSpec("wide_f32", 32768, 40960, dtype="f32", seed=71, tensor_id=4,
                            dist=DIST_STUDENT_T3), [AUTO, VECTOR]),
}


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    free, _ = torch.cuda.mem_get_info()
    if free < 24 << 30:
        pytest.skip("needs 24 GB of free device memory")
    yield
    torch.cuda.synchronize()
    torch.cuda.empty_cache()


@pytest.mark.parametrize("name", list(CASES))
def test_at_4gib_and_beyond(name):
    sp, paths = CASES[name]
    assert sp.numel_storage * sp.elem_bytes >= (4 << 30) - 256   # offsets need 64 bits
    x = W.materialize(sp)
    xdev = torch.from_numpy(x.view(np.uint8)).cuda()
    rng = np.random.default_rng(17)
    first = None
    try:
        for path in paths:
            (out,) = run([sp], [xdev.data_ptr()], path)
            assert out.y.canaries_intact() and out.s.canaries_intact(), (name, path)
            assert no_nan_codes(out), (name, path)
            assert check_sampled(sp, x, out, rng, k=6) >= 4
            if first is None:
                first = out
            else:
                assert torch.equal(out.y.view, first.y.view), (name, path)
                assert torch.equal(out.s.view, first.s.view), (name, path)
                del out
        if name == "wide":
            dequantize_and_check(sp, x, first, rng)
    finally:
        del xdev, first
        torch.cuda.empty_cache()


def dequantize_and_check(sp, x, q, rng):
    """bf16 dequantization of the whole 5.4 GB output; sampled blocks against
    the oracle's dequantization of the oracle's own codes (equal to the GPU's
    there, as check_sampled has shown)."""
    out = Guarded(sp.numel * 2)
    st = fq.fp8bq_dequantize(q.y.ptr, q.s.ptr, 1, sp.M, sp.N, *sp.block, out.ptr,
                             fq.FP8BQ_BF16, sp.N, 0)
    assert st == fq.FP8BQ_OK and fq.fp8bq_sync_status() == fq.FP8BQ_OK
    assert out.canaries_intact()
    bm, bn = sp.block
    ov = out.view.view(torch.int16).view(sp.M, sp.N)
    for _, bi, bj in sample_blocks(sp, rng, 4):
        yw, sw = oracle.quantize_block(x, sp.M, sp.N, sp.row_stride, bm, bn, bi, bj)
        want = oracle.dequantize(yw, np.array([[sw]], np.float32), bm, bn, "bf16")
        got = ov[bi * bm:bi * bm + yw.shape[0], bj * bn:bj * bn + yw.shape[1]].cpu().numpy()
        assert np.array_equal(got.view(np.uint16), want), (bi, bj)
