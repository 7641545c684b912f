"""Stream order under programmatic dependent launch: every kernel of the
library may be scheduled while the previous kernel of its stream drains, but
waits for it before touching memory.  A chain on one stream (a PyTorch kernel
writes the input, the quantizer reads it, the dequantizer reads the codes, a
PyTorch kernel reads the dequantized weights, the per-tensor scale reads the
input again), repeated with the input rewritten every time, must give the
oracle's result at every link, with the launch mode on and off."""
import numpy as np
import pytest
import torch

import blockwise_fp8_weight_b200 as fq
import oracle
from synth import DIST_STUDENT_T3, TensorSpec
from synth import workloads as W

pytestmark = pytest.mark.gpu

M, N = 1000, 2048


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    yield
    torch.cuda.synchronize()


@pytest.mark.parametrize("pdl", [1, 0])
def test_chain_keeps_stream_order(pdl):
    specs = [TensorSpec(f"pdl.{k}", M, N, seed=90 + k, tensor_id=k, dist=DIST_STUDENT_T3)
             for k in range(2)]
    host = [W.materialize(sp) for sp in specs]
    src = [torch.from_numpy(h.view(np.int16).reshape(M, N)).cuda().view(torch.bfloat16)
           for h in host]
    want = [oracle.quantize(h, M, N, N, 128, 128) for h in host]
    want_z = [oracle.dequantize(y, s, 128, 128, "bf16") for y, s in want]
    want_sc = [oracle.tensor_scale(h) for h in host]

    x = torch.empty_like(src[0])
    outs = []
    assert fq.fp8bq_set_pdl(pdl) == fq.FP8BQ_OK
    try:
        for k in range(16):
            x.copy_(src[k % 2])                               # PyTorch writes the input
            y, s = fq.scaled_fp8_blockwise(x, [128, 128])     # ours reads it
            z = fq.dequantize_fp8_blockwise(y, s)             # ours reads ours
            zmax = z.float().abs().amax()                     # PyTorch reads ours
            sc = fq.tensor_scales([x])                        # zero, amax, finalize kernels
            outs.append((y, s, z, zmax, sc))
        torch.cuda.synchronize()
    finally:
        fq.fp8bq_set_pdl(1)
    assert fq.fp8bq_sync_status(None) == fq.FP8BQ_OK
    for k, (y, s, z, zmax, sc) in enumerate(outs):
        wy, ws = want[k % 2]
        assert np.array_equal(y.view(torch.uint8).cpu().numpy(), wy), f"codes of link {k}"
        assert np.array_equal(s.cpu().numpy().view(np.uint32), ws.view(np.uint32)), \
            f"descales of link {k}"
        zb = z.view(torch.int16).cpu().numpy().view(np.uint16)
        assert np.array_equal(zb, want_z[k % 2]), f"dequantized weights of link {k}"
        wmax = np.abs((want_z[k % 2].astype(np.uint32) << 16).view(np.float32)).max()
        assert float(zmax) == float(wmax), f"PyTorch read of link {k}"
        assert sc.cpu().numpy().view(np.uint32)[0] == np.float32(want_sc[k % 2]).view(np.uint32), \
            f"tensor scale of link {k}"
