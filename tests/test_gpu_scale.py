"""GPU parity of the per-tensor scale kernel (max(max|x|, eps) / 448) against
the oracle, bit for bit, through the C ABI, on activation-shaped tensors of
both dtypes, ragged and misaligned sizes, all-zero and empty tensors."""
import numpy as np
import pytest
import torch

import blockwise_fp8_weight_b200 as fq
import oracle
from synth import DIST_STUDENT_T3, TensorSpec
from synth import workloads as W
from tests.gpu_util import Guarded, to_device

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    yield
    torch.cuda.synchronize()


def test_tensor_scales_match_oracle():
    specs = [
        TensorSpec("q", 8192, 4096, seed=95, tensor_id=1, sigma=1.0, row_lognormal_sigma=1.0),
        TensorSpec("k", 8192, 1024, seed=95, tensor_id=2, sigma=1.0, row_lognormal_sigma=1.0),
        TensorSpec("v", 8192, 1024, dtype="f32", seed=95, tensor_id=3, dist=DIST_STUDENT_T3),
        TensorSpec("ragged", 1, 4097 * 3 + 5, seed=95, tensor_id=4, dist=DIST_STUDENT_T3),
        TensorSpec("tiny", 1, 7, dtype="f32", seed=95, tensor_id=5),
    ]
    hosts = [W.materialize(sp) for sp in specs]
    devs = [to_device(x, offset_bytes=(2 if i == 3 else 0)) for i, x in enumerate(hosts)]
    zeros = torch.zeros(5000, dtype=torch.bfloat16, device="cuda")
    descs = []
    for sp, (owner, ptr) in zip(specs, devs):
        d = fq.fp8bq_scale_desc()
        d.x, d.numel = ptr, sp.numel
        d.dtype_in = fq.FP8BQ_BF16 if sp.dtype == "bf16" else fq.FP8BQ_F32
        d.reserved = 0
        descs.append(d)
    z = fq.fp8bq_scale_desc()
    z.x, z.numel, z.dtype_in = zeros.data_ptr(), zeros.numel(), fq.FP8BQ_BF16
    e = fq.fp8bq_scale_desc()
    e.x, e.numel, e.dtype_in = 0, 0, fq.FP8BQ_F32
    descs += [z, e]
    out = Guarded(4 * len(descs))
    assert fq.fp8bq_tensor_scale(descs, out.ptr) == fq.FP8BQ_OK
    assert fq.fp8bq_sync_status() == fq.FP8BQ_OK
    assert out.canaries_intact()
    got = out.numpy().view(np.float32)
    want = [oracle.tensor_scale(x) for x in hosts]
    floor = oracle.tensor_scale(np.zeros(1, dtype=np.float32))
    want += [floor, floor]
    assert np.array_equal(got.view(np.uint32), np.array(want, dtype=np.float32).view(np.uint32))


def test_tensor_scales_python_api():
    x = torch.randn(4096, 512, device="cuda").to(torch.bfloat16) * 3
    y = torch.randn(1000, device="cuda")
    s = fq.tensor_scales([x, y])
    torch.cuda.synchronize()
    xn = x.view(torch.int16).cpu().numpy().view(np.uint16)
    assert s[0].item() == oracle.tensor_scale(xn)
    assert s[1].item() == oracle.tensor_scale(y.cpu().numpy())
