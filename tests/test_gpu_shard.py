"""The shard-quantize + all-gather path on the GPU with one NCCL rank: the
CUDA quantizer on the shard, the gather through NCCL, and the result equal to
the oracle's quantization of the whole weight.  (More ranks need more GPUs
than one test run has; the multi-rank host logic is covered on gloo ranks in
test_shard_host.py.)"""
import os
import socket

import numpy as np
import pytest
import torch

import oracle
from synth import DIST_STUDENT_T3, TensorSpec
from synth import workloads as W

pytestmark = pytest.mark.gpu


def _port() -> int:
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def test_quantize_and_allgather_one_rank():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import torch.distributed as dist
    from blockwise_fp8_weight_b200.shard import quantize_and_allgather
    M, N = 1000, 384
    sp = TensorSpec("shard.gpu", M, N, seed=19, tensor_id=3, dist=DIST_STUDENT_T3)
    x = W.materialize(sp)
    xt = torch.from_numpy(x.view(np.int16).reshape(M, N)).cuda().view(torch.bfloat16)
    store = dist.TCPStore("127.0.0.1", _port(), 1, True)
    dist.init_process_group("nccl", store=store, rank=0, world_size=1,
                            device_id=torch.device("cuda", torch.cuda.current_device()))
    try:
        y, s = quantize_and_allgather(xt, M, (128, 128))
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    wy, ws = oracle.quantize(x, M, N, N, 128, 128)
    assert y.dtype == torch.float8_e4m3fn and tuple(y.shape) == (M, N)
    assert np.array_equal(y.view(torch.uint8).cpu().numpy(), wy)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), ws.view(np.uint32))
