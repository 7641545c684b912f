"""Quantize a row-sharded weight on every rank, then all-gather the e4m3fn
codes and descales (one process per GPU, ``torch.distributed``).

The idea is the one the verl FSDP sharding-manager page raises (issue #1803:
whether the parameter all-gather could be fused with FP8 quantization to cut
its memory and traffic): quantize each rank's shard before the gather, so
that 1 byte per element plus one fp32 descale per block crosses NVLink instead
of the 2 bytes per element of bf16.  Blocks are independent, so quantizing row
shards whose boundaries fall on block rows yields exactly the bytes of
quantizing the whole matrix.

Shards are whole block rows (``shard_rows``): rank r holds rows
[r * R, min((r + 1) * R, M)) of the [M, N] weight, R a multiple of block_m.
A shard boundary inside a block row would need the boundary rows exchanged
before quantizing; such shardings are refused.

This module is collective plumbing only: the quantization itself is the
library's CUDA kernel (``scaled_fp8_blockwise``).
"""
from __future__ import annotations

from typing import Sequence


def shard_rows(M: int, world: int, block_m: int) -> list[tuple[int, int]]:
    """Row range [lo, hi) of every rank: whole block rows, ceil(gm / world)
    of them per rank (gm = ceil(M / block_m)), so the last ranks may hold
    fewer rows or none."""
    if M < 0 or world < 1 or block_m < 1:
        raise ValueError("need M >= 0, world >= 1, block_m >= 1")
    gm = -(-M // block_m)
    per = -(-gm // world) * block_m
    return [(min(r * per, M), min((r + 1) * per, M)) for r in range(world)]


def gather_quantized_shards(codes, descale, M: int, N: int,
                            weight_block_size: Sequence[int] = (128, 128), group=None):
    """All-gather every rank's quantized shard into the whole weight.

    ``codes``: this rank's [hi - lo, N] e4m3fn codes (``torch.uint8`` or
    ``torch.float8_e4m3fn``) for its rows [lo, hi) of ``shard_rows(M, world,
    block_m)``; ``descale``: its [ceil((hi - lo) / block_m), ceil(N / block_n)]
    fp32 descales.  Every rank must call this with the same M, N and block.
    Returns ``(codes [M, N], descale [ceil(M / block_m), ceil(N / block_n)])``
    on every rank, codes in the input's dtype, on the input's device.
    """
    import torch
    import torch.distributed as dist

    bm, bn = (int(b) for b in weight_block_size)
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    ranges = shard_rows(M, world, bm)
    lo, hi = ranges[rank]
    gm, gn = -(-M // bm), -(-N // bn)
    if tuple(codes.shape) != (hi - lo, N):
        raise ValueError(f"rank {rank}: codes are {tuple(codes.shape)}, expected {(hi - lo, N)} "
                         f"(rows {lo}..{hi} of shard_rows({M}, {world}, {bm}))")
    if tuple(descale.shape) != (-(-(hi - lo) // bm), gn) or descale.dtype != torch.float32:
        raise ValueError(f"rank {rank}: descale is {tuple(descale.shape)} {descale.dtype}, "
                         f"expected {(-(-(hi - lo) // bm), gn)} float32")
    if M == 0 or N == 0:  # the same on every rank: no collective
        return codes.new_empty((M, N)), descale.new_empty((gm, gn))
    rows = -(-gm // world) * bm  # rows of an unclipped shard (a multiple of bm)
    dev = codes.device
    # equal-sized pieces for the gather: short shards are padded, then trimmed
    pc = torch.zeros((rows, N), dtype=torch.uint8, device=dev)
    pc[:hi - lo] = codes.view(torch.uint8)
    ps = torch.zeros((rows // bm, gn), dtype=torch.float32, device=dev)
    ps[:descale.shape[0]] = descale
    all_c = [torch.empty_like(pc) for _ in range(world)]
    all_s = [torch.empty_like(ps) for _ in range(world)]
    dist.all_gather(all_c, pc, group=group)
    dist.all_gather(all_s, ps, group=group)
    full_c = torch.cat(all_c)[:M].contiguous()
    full_s = torch.cat(all_s)[:gm].contiguous()
    return full_c.view(codes.dtype), full_s


def quantize_and_allgather(shard, M: int, weight_block_size: Sequence[int] = (128, 128),
                           group=None, stream=None):
    """Quantize this rank's row shard of an [M, N] weight with the library's
    CUDA kernel, then all-gather codes and descales.

    ``shard`` is this rank's rows [lo, hi) of ``shard_rows(M, world,
    block_m)`` as a CUDA tensor [hi - lo, N] (bf16 or fp32, unit stride along
    N).  Returns ``(fp8_data [M, N] float8_e4m3fn, descale [ceil(M / block_m),
    ceil(N / block_n)] fp32)`` on every rank, byte for byte what
    ``scaled_fp8_blockwise`` gives on the whole weight.
    """
    import contextlib

    import torch

    from . import scaled_fp8_blockwise
    block = tuple(int(b) for b in weight_block_size)
    # quantize and gather on one stream, so that the collective (ordered after
    # the current stream's work) sees the finished codes
    ctx = torch.cuda.stream(stream) if stream is not None else contextlib.nullcontext()
    with ctx:
        codes, descale = scaled_fp8_blockwise(shard, block)
        return gather_quantized_shards(codes, descale, M, int(shard.shape[-1]), block, group)
