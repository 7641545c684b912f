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

Data movement: the gather output is one buffer of ``world`` equal slots of R
rows (``GatherBuffers``); rank r's slot is where its shard's codes go, so the
library's kernel writes them there directly and the all-gather runs in place
(each rank sends its own slot).  The whole weight is then the first M rows of
the buffer: a view, with no concatenation or copy.

This module is collective plumbing only: the quantization itself is the
library's CUDA kernel.
"""
from __future__ import annotations

from dataclasses import dataclass
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


@dataclass
class GatherBuffers:
    """Outputs of one gathered weight.

    ``codes`` [world * R, N] uint8 and ``descale`` [world * R / block_m, gn]
    fp32, R the rows of an unclipped shard; rank r's slot is rows
    [r * R, (r + 1) * R) of ``codes`` and block rows [r * R / block_m, ...)
    of ``descale``.  Slot rows past M are padding and never read back."""
    codes: object
    descale: object
    M: int
    N: int
    rows: int          # R
    block: tuple[int, int]

    @property
    def gm(self) -> int:
        return -(-self.M // self.block[0])

    def slot(self, rank: int, lo: int, hi: int):
        """This rank's part of the slot: (codes [hi - lo, N], descale
        [ceil((hi - lo) / block_m), gn]) views."""
        bm = self.block[0]
        r0, b0 = rank * self.rows, rank * self.rows // bm
        return (self.codes[r0:r0 + hi - lo], self.descale[b0:b0 + -(-(hi - lo) // bm)])

    def whole(self):
        """(codes [M, N], descale [gm, gn]) views of the gathered weight."""
        return self.codes[:self.M], self.descale[:self.gm]


def gather_buffers(M: int, N: int, weight_block_size: Sequence[int], world: int,
                   device) -> GatherBuffers:
    """Allocate the gather outputs of an [M, N] weight for ``world`` ranks."""
    import torch
    bm, bn = (int(b) for b in weight_block_size)
    gm, gn = -(-M // bm), -(-N // bn)
    rows = -(-gm // world) * bm
    codes = torch.empty((world * rows, N), dtype=torch.uint8, device=device)
    descale = torch.empty((world * rows // bm, gn), dtype=torch.float32, device=device)
    return GatherBuffers(codes, descale, M, N, rows, (bm, bn))


def _gather_in_place(buf: GatherBuffers, rank: int, group) -> None:
    """All-gather every rank's slot into every rank's buffer (each rank sends
    its own slot of the output, so nothing is staged)."""
    import torch.distributed as dist
    bm = buf.block[0]
    per_c, per_s = buf.rows, buf.rows // bm
    dist.all_gather_into_tensor(buf.codes, buf.codes[rank * per_c:(rank + 1) * per_c],
                                group=group)
    dist.all_gather_into_tensor(buf.descale, buf.descale[rank * per_s:(rank + 1) * per_s],
                                group=group)


def _check_shard(what, rank, shape, want) -> None:
    if tuple(shape) != tuple(want):
        raise ValueError(f"rank {rank}: {what} {tuple(shape)}, expected {tuple(want)}")


def gather_quantized_shards(codes, descale, M: int, N: int,
                            weight_block_size: Sequence[int] = (128, 128), group=None):
    """All-gather every rank's quantized shard into the whole weight.

    ``codes``: this rank's [hi - lo, N] e4m3fn codes (``torch.uint8`` or
    ``torch.float8_e4m3fn``) for its rows [lo, hi) of ``shard_rows(M, world,
    block_m)``; ``descale``: its [ceil((hi - lo) / block_m), ceil(N / block_n)]
    fp32 descales.  Every rank must call this with the same M, N and block.
    Returns ``(codes [M, N], descale [ceil(M / block_m), ceil(N / block_n)])``
    on every rank, codes in the input's dtype, on the input's device (views
    of the gather buffer).  The shard is copied once, into its slot; callers
    that can quantize straight into the slot use ``quantize_and_allgather``.
    """
    import torch
    import torch.distributed as dist

    bm, bn = (int(b) for b in weight_block_size)
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    lo, hi = shard_rows(M, world, bm)[rank]
    gm, gn = -(-M // bm), -(-N // bn)
    _check_shard("codes are", rank, codes.shape, (hi - lo, N))
    _check_shard("descale is", rank, descale.shape, (-(-(hi - lo) // bm), gn))
    if descale.dtype != torch.float32:
        raise ValueError(f"rank {rank}: descale is {descale.dtype}, expected float32")
    if M == 0 or N == 0:  # the same on every rank: no collective
        return codes.new_empty((M, N)), descale.new_empty((gm, gn))
    buf = gather_buffers(M, N, (bm, bn), world, codes.device)
    yc, sc = buf.slot(rank, lo, hi)
    yc.copy_(codes.view(torch.uint8))
    sc.copy_(descale)
    _gather_in_place(buf, rank, group)
    y, s = buf.whole()
    return y.view(codes.dtype), s


def quantize_and_allgather(shard, M: int, weight_block_size: Sequence[int] = (128, 128),
                           group=None, stream=None):
    """Quantize this rank's row shard of an [M, N] weight with the library's
    CUDA kernel, straight into its slot of the gather buffer, then all-gather
    codes and descales in place.

    ``shard`` is this rank's rows [lo, hi) of ``shard_rows(M, world,
    block_m)`` as a CUDA tensor [hi - lo, N] (bf16 or fp32, unit stride along
    N).  Returns ``(fp8_data [M, N] float8_e4m3fn, descale [ceil(M / block_m),
    ceil(N / block_n)] fp32)`` on every rank, byte for byte what
    ``scaled_fp8_blockwise`` gives on the whole weight.
    """
    import contextlib

    import torch
    import torch.distributed as dist

    from . import check, fp8bq_quantize_batched, make_desc
    block = tuple(int(b) for b in weight_block_size)
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    N = int(shard.shape[-1])
    lo, hi = shard_rows(M, world, block[0])[rank]
    _check_shard("the shard is", rank, shard.shape, (hi - lo, N))
    gm, gn = -(-M // block[0]), -(-N // block[1])
    # quantize and gather on one stream, so that the collective (ordered after
    # the current stream's work) sees the finished codes; the buffers are
    # allocated on that stream too
    ctx = torch.cuda.stream(stream) if stream is not None else contextlib.nullcontext()
    with ctx:
        if M == 0 or N == 0:
            return (torch.empty((M, N), dtype=torch.float8_e4m3fn, device=shard.device),
                    torch.empty((gm, gn), dtype=torch.float32, device=shard.device))
        buf = gather_buffers(M, N, block, world, shard.device)
        if hi > lo:
            yc, sc = buf.slot(rank, lo, hi)
            check(fp8bq_quantize_batched([make_desc(shard, yc, sc, block)]),
                  "quantize_and_allgather")
        _gather_in_place(buf, rank, group)
        y, s = buf.whole()
        return y.view(torch.float8_e4m3fn), s
