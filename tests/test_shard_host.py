"""Host logic of the shard-quantize + all-gather path on gloo ranks (CPU): the
row split into whole block rows, and the gather that reassembles codes and
descales.  Each rank's shard is quantized by the oracle here (the CUDA
quantizer needs a GPU); the reassembled weight must equal the oracle's
quantization of the whole matrix, byte for byte -- which also checks that
block-row shards quantize independently."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import oracle  # noqa: E402
from blockwise_fp8_weight_b200.shard import gather_quantized_shards, shard_rows  # noqa: E402
from synth import DIST_STUDENT_T3, TensorSpec  # noqa: E402
from synth import workloads as W  # noqa: E402


def test_shard_rows_cover_whole_block_rows():
    for M, world, bm in [(1000, 2, 128), (1000, 3, 128), (200, 3, 128), (7, 4, 1), (0, 2, 128),
                         (4096, 8, 128), (130, 5, 64), (1, 1, 128)]:
        r = shard_rows(M, world, bm)
        assert len(r) == world
        assert r[0][0] == 0 and r[-1][1] == M
        for (lo, hi), (lo2, _) in zip(r, r[1:]):
            assert hi == lo2 and lo <= hi          # contiguous, in order
        for lo, hi in r:
            assert lo % bm == 0 or lo == M          # every shard starts on a block row
        per = r[0][1] - r[0][0]
        assert all(hi - lo <= per for lo, hi in r)
    with pytest.raises(ValueError):
        shard_rows(10, 0, 128)


def _port() -> int:
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _rank(rank, world, port, case, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        M, N, block, dtype = case
        sp = TensorSpec("shard", M, N, dtype=dtype, block=block, seed=17, tensor_id=M * 7 + N,
                        dist=DIST_STUDENT_T3)
        x = W.materialize(sp).reshape(M, N)
        lo, hi = shard_rows(M, world, block[0])[rank]
        local = np.ascontiguousarray(x[lo:hi])
        if hi > lo:
            y, s = oracle.quantize(local, hi - lo, N, N, *block)
        else:
            y = np.zeros((0, N), np.uint8)
            s = np.zeros((0, -(-N // block[1])), np.float32)
        fy, fs = gather_quantized_shards(torch.from_numpy(y), torch.from_numpy(s), M, N, block)
        wy, ws = oracle.quantize(np.ascontiguousarray(x), M, N, N, *block)
        ok = (fy.shape == (M, N) and np.array_equal(fy.numpy(), wy)
              and np.array_equal(fs.numpy().view(np.uint32), ws.view(np.uint32))
              # the results are the leading rows of the (padded) gather
              # buffers, not copies
              and fy.untyped_storage().nbytes() > fy.numel()
              and fy.data_ptr() == fy.untyped_storage().data_ptr()
              and fs.data_ptr() == fs.untyped_storage().data_ptr()
              and fy.is_contiguous() and fs.is_contiguous())
        q.put((rank, ok))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,case", [
    (2, (1000, 384, (128, 128), "bf16")),   # ragged last block row
    (3, (1000, 384, (128, 128), "f32")),
    (3, (200, 130, (128, 128), "bf16")),    # third rank holds no rows; ragged columns
    (2, (37, 256, (1, 128), "bf16")),       # 1x128 blocks: any row boundary is a block row
    (2, (100, 256, (128, 128), "bf16")),    # one block row: rank 0's shard is clipped at M
])
def test_gather_reassembles_the_whole_quantized_weight(world, case):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, case, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert res == [(r, True) for r in range(world)]


def test_gather_refuses_a_wrong_shard_shape():
    import torch.distributed as dist
    port = _port()
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=0, world_size=1)
    try:
        with pytest.raises(ValueError, match="codes are"):
            gather_quantized_shards(torch.zeros(5, 8, dtype=torch.uint8),
                                    torch.zeros(1, 1, dtype=torch.float32), 6, 8)
        with pytest.raises(ValueError, match="descale is"):
            gather_quantized_shards(torch.zeros(6, 8, dtype=torch.uint8),
                                    torch.zeros(2, 1, dtype=torch.float32), 6, 8)
        y, s = gather_quantized_shards(torch.zeros(6, 8, dtype=torch.uint8),
                                       torch.ones(1, 1, dtype=torch.float32), 6, 8)
        assert y.shape == (6, 8) and s.shape == (1, 1) and float(s[0, 0]) == 1.0
    finally:
        dist.destroy_process_group()


def _rank_rows(rank, world, port, case, q):
    """Rows split anywhere: halo exchange, oracle quantization of this rank's
    block rows, broadcast assembly."""
    import torch.distributed as dist
    from blockwise_fp8_weight_b200.shard import (broadcast_quantized, exchange_halo,
                                                 owned_block_rows)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        M, N, block, dtype, ranges = case
        sp = TensorSpec("rows", M, N, dtype=dtype, block=block, seed=29, tensor_id=M * 5 + N,
                        dist=DIST_STUDENT_T3)
        x = W.materialize(sp).reshape(M, N)
        lo, hi = ranges[rank]
        # bf16 bit patterns travel as int16 (the same bytes; gloo has no uint16)
        wire = np.int16 if dtype == "bf16" else np.float32
        rows, kb, ke = exchange_halo(torch.from_numpy(np.ascontiguousarray(x[lo:hi]).view(wire)),
                                     ranges, M, block[0])
        rows = rows.numpy().view(x.dtype)
        assert (kb, ke) == owned_block_rows(ranges, rank, block[0])
        r0, r1 = kb * block[0], min(ke * block[0], M)
        ok = np.array_equal(rows, x[r0:r1]) if r1 > r0 else rows.shape[0] == 0
        gn = -(-N // block[1])
        if r1 > r0:
            y, s = oracle.quantize(np.ascontiguousarray(rows), r1 - r0, N, N, *block)
        else:
            y, s = np.zeros((0, N), np.uint8), np.zeros((0, gn), np.float32)
        fy, fs = broadcast_quantized(torch.from_numpy(y), torch.from_numpy(s), ranges, M, N, block)
        wy, ws = oracle.quantize(np.ascontiguousarray(x), M, N, N, *block)
        ok = ok and np.array_equal(fy.numpy(), wy) and \
            np.array_equal(fs.numpy().view(np.uint32), ws.view(np.uint32))
        q.put((rank, bool(ok)))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,case", [
    (3, (1000, 256, (128, 128), "bf16", None)),            # even split: 334 rows per rank
    (2, (300, 130, (128, 128), "f32", [(0, 5), (5, 300)])),  # a head of 123 rows
    (4, (300, 256, (128, 128), "bf16", [(0, 100), (100, 120), (120, 250), (250, 300)])),
    (3, (200, 256, (64, 64), "bf16", [(0, 64), (64, 64), (64, 200)])),  # an empty rank
    (3, (90, 256, (32, 128), "bf16", [(0, 33), (33, 34), (34, 90)])),   # one-row rank
])
def test_rows_split_anywhere_reassemble_exactly(world, case):
    from blockwise_fp8_weight_b200.shard import row_chunks
    M, N, block, dtype, ranges = case
    case = (M, N, block, dtype, ranges or row_chunks(M, world))
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _port()
    procs = [ctx.Process(target=_rank_rows, args=(r, world, port, case, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert res == [(r, True) for r in range(world)]


def test_row_ranges_are_checked():
    from blockwise_fp8_weight_b200.shard import _check_ranges, owned_block_rows, row_chunks
    assert row_chunks(1000, 3) == [(0, 334), (334, 668), (668, 1000)]
    assert row_chunks(2, 4) == [(0, 1), (1, 2), (2, 2), (2, 2)]
    with pytest.raises(ValueError):
        _check_ranges([(0, 5), (6, 10)], 10, 2)            # a gap
    with pytest.raises(ValueError):
        _check_ranges([(0, 5), (5, 9)], 10, 2)             # short of M
    r = [(0, 100), (100, 120), (120, 250), (250, 300)]
    assert [owned_block_rows(r, k, 128) for k in range(4)] == [(0, 1), (1, 1), (1, 2), (2, 3)]
