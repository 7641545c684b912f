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


def test_sharded_quant_gather_many_weights_one_rank():
    """ShardedQuantGather: one grouped quantize launch over every weight's
    shard into its gather slot, then the in-place gathers; twice on the same
    buffers (a sync every RL step), each time byte-exact against the oracle."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import torch.distributed as dist
    from blockwise_fp8_weight_b200.shard import ShardedQuantGather
    specs = [TensorSpec(f"sqg.{i}", M, N, seed=23, tensor_id=i, dist=DIST_STUDENT_T3)
             for i, (M, N) in enumerate([(1000, 384), (256, 4096), (130, 1024), (0, 256)])]
    hosts = [W.materialize(sp) for sp in specs]
    xs = [torch.from_numpy(x.view(np.int16).reshape(sp.M, sp.N)).cuda().view(torch.bfloat16)
          for sp, x in zip(specs, hosts)]
    store = dist.TCPStore("127.0.0.1", _port(), 1, True)
    dist.init_process_group("nccl", store=store, rank=0, world_size=1,
                            device_id=torch.device("cuda", torch.cuda.current_device()))
    try:
        sqg = ShardedQuantGather([(sp.M, sp.N) for sp in specs], (128, 128))
        for _ in range(2):
            out = sqg.run(xs)
            torch.cuda.synchronize()
            for sp, x, (y, s) in zip(specs, hosts, out):
                wy, ws = oracle.quantize(x, sp.M, sp.N, sp.N, 128, 128)
                assert y.dtype == torch.float8_e4m3fn and tuple(y.shape) == (sp.M, sp.N)
                assert np.array_equal(y.view(torch.uint8).cpu().numpy(), wy)
                assert np.array_equal(s.cpu().numpy().view(np.uint32), ws.view(np.uint32))
            for b in sqg.bufs:                       # the second run rewrites every byte
                b.codes.fill_(0x7F)
                b.descale.fill_(float("nan"))
    finally:
        dist.destroy_process_group()


def test_quantize_and_allgather_rows_one_rank():
    """The any-row-split path on the GPU with one NCCL rank: the halo exchange
    has nothing to move, the library quantizes the rank's block rows and the
    broadcast assembles the weight, byte-exact against the oracle."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import torch.distributed as dist
    from blockwise_fp8_weight_b200.shard import quantize_and_allgather_rows, row_chunks
    M, N = 1000, 384
    sp = TensorSpec("rows.gpu", M, N, seed=31, tensor_id=4, dist=DIST_STUDENT_T3)
    x = W.materialize(sp)
    xt = torch.from_numpy(x.view(np.int16).reshape(M, N)).cuda().view(torch.bfloat16)
    store = dist.TCPStore("127.0.0.1", _port(), 1, True)
    dist.init_process_group("nccl", store=store, rank=0, world_size=1,
                            device_id=torch.device("cuda", torch.cuda.current_device()))
    try:
        y, s = quantize_and_allgather_rows(xt, row_chunks(M, 1), M, (128, 128))
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    wy, ws = oracle.quantize(x, M, N, N, 128, 128)
    assert y.dtype == torch.float8_e4m3fn and tuple(y.shape) == (M, N)
    assert np.array_equal(y.view(torch.uint8).cpu().numpy(), wy)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), ws.view(np.uint32))
