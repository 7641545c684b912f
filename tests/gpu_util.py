"""Helpers for the GPU parity tests: guarded device buffers, runs through the
C ABI, and the oracle's expected outputs for a workload tensor."""
from __future__ import annotations

import numpy as np
import torch

import blockwise_fp8_weight_b200 as fq
import oracle
from synth import TensorSpec

GUARD = 4096          # bytes of canary before and after every output buffer
CANARY = 0xA5


class Guarded:
    """A device buffer with canary bands on both sides (the library must write
    exactly the bytes it owns)."""

    def __init__(self, nbytes: int, offset: int = 0):
        self.nbytes = nbytes
        self.offset = offset
        self.raw = torch.full((nbytes + offset + 2 * GUARD,), CANARY, dtype=torch.uint8,
                              device="cuda")
        self.view = self.raw[GUARD + offset:GUARD + offset + nbytes]

    @property
    def ptr(self) -> int:
        return self.raw.data_ptr() + GUARD + self.offset

    def canaries_intact(self) -> bool:
        head = self.raw[:GUARD + self.offset]
        tail = self.raw[GUARD + self.offset + self.nbytes:]
        return bool((head == CANARY).all().item()) and bool((tail == CANARY).all().item())

    def numpy(self) -> np.ndarray:
        return self.view.cpu().numpy()


def to_device(x: np.ndarray, offset_bytes: int = 0) -> tuple[torch.Tensor, int]:
    """Upload a host array; returns (owner tensor, pointer).  With an offset the
    data starts that many bytes past a 256-byte-aligned base."""
    raw = torch.empty(x.nbytes + offset_bytes + 256, dtype=torch.uint8, device="cuda")
    base = raw.data_ptr() + offset_bytes
    view = raw[offset_bytes:offset_bytes + x.nbytes]
    view.copy_(torch.from_numpy(x.view(np.uint8).reshape(-1)))
    return raw, base


class Outputs:
    def __init__(self, spec: TensorSpec, y_offset: int = 0):
        gm, gn = spec.grid
        self.spec = spec
        self.y = Guarded(spec.numel, y_offset)
        self.s = Guarded(spec.batch * gm * gn * 4)

    def desc(self, x_ptr: int) -> fq.fp8bq_desc:
        sp = self.spec
        gm, gn = sp.grid
        d = fq.fp8bq_desc()
        d.x, d.y_u8, d.descale_f32 = x_ptr, self.y.ptr, self.s.ptr
        d.M, d.N, d.ld = sp.M, sp.N, sp.row_stride
        d.batch = sp.batch
        d.x_batch_stride = sp.batch_stride
        d.y_batch_stride = sp.M * sp.N
        d.s_batch_stride = gm * gn
        d.dtype_in = fq.FP8BQ_BF16 if sp.dtype == "bf16" else fq.FP8BQ_F32
        d.block_m, d.block_n = sp.block
        d.reserved = 0
        return d

    def result(self) -> tuple[np.ndarray, np.ndarray]:
        sp = self.spec
        gm, gn = sp.grid
        assert self.y.canaries_intact(), f"{sp.name}: bytes written outside y"
        assert self.s.canaries_intact(), f"{sp.name}: bytes written outside descale"
        y = self.y.numpy().reshape(sp.batch, sp.M, sp.N)
        s = self.s.numpy().view(np.float32).reshape(sp.batch, gm, gn)
        return y, s


def run(specs, x_ptrs, path=fq.FP8BQ_PATH_AUTO, y_offsets=None, stream=None):
    """Quantize all specs in one batched call; returns the Outputs."""
    outs = [Outputs(sp, 0 if y_offsets is None else y_offsets[i]) for i, sp in enumerate(specs)]
    descs = [o.desc(p) for o, p in zip(outs, x_ptrs)]
    assert fq.fp8bq_set_path(path) == fq.FP8BQ_OK
    try:
        st = fq.fp8bq_quantize_batched(descs, stream=stream)
        assert st == fq.FP8BQ_OK, fq.fp8bq_status_string(st)
        st = fq.fp8bq_sync_status(stream)
        assert st == fq.FP8BQ_OK, fq.fp8bq_status_string(st)
    finally:
        fq.fp8bq_set_path(fq.FP8BQ_PATH_AUTO)
    return outs


def oracle_expected(spec: TensorSpec, x: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """Oracle output for every matrix of the spec: y [batch, M, N], s [batch, gm, gn]."""
    gm, gn = spec.grid
    ys = np.empty((spec.batch, spec.M, spec.N), dtype=np.uint8)
    ss = np.empty((spec.batch, gm, gn), dtype=np.float32)
    for b in range(spec.batch):
        xb = x[b * spec.batch_stride:(b + 1) * spec.batch_stride]
        ys[b], ss[b] = oracle.quantize(np.ascontiguousarray(xb), spec.M, spec.N, spec.row_stride,
                                       *spec.block)
    return ys, ss


def assert_same(spec: TensorSpec, got, want) -> None:
    yg, sg = got
    yw, sw = want
    bad = np.flatnonzero(yg.reshape(-1) != yw.reshape(-1))
    assert bad.size == 0, (f"{spec.name}: {bad.size} e4m3 bytes differ; first at flat index "
                           f"{bad[0]}: got {yg.reshape(-1)[bad[0]]:#04x} want "
                           f"{yw.reshape(-1)[bad[0]]:#04x}")
    sb = np.flatnonzero(sg.view(np.uint32).reshape(-1) != sw.view(np.uint32).reshape(-1))
    assert sb.size == 0, (f"{spec.name}: {sb.size} descales differ; first at {sb[0]}: got "
                          f"{sg.reshape(-1)[sb[0]]!r} want {sw.reshape(-1)[sb[0]]!r}")


def sample_blocks(sp: TensorSpec, rng, k=6):
    gm, gn = sp.grid
    picks = {(0, 0, 0), (sp.batch - 1, gm - 1, gn - 1), (0, 0, gn - 1), (sp.batch - 1, gm - 1, 0)}
    for _ in range(k):
        picks.add((int(rng.integers(sp.batch)), int(rng.integers(gm)), int(rng.integers(gn))))
    return sorted(picks)


def check_sampled(sp: TensorSpec, x: np.ndarray, out: Outputs, rng, k=6) -> int:
    """Compare sampled blocks of a device output with the oracle, block by block."""
    gm, gn = sp.grid
    bm, bn = sp.block
    yv = out.y.view.view(sp.batch, sp.M, sp.N)
    sv = out.s.view.view(torch.float32).view(sp.batch, gm, gn)
    n = 0
    for b, bi, bj in sample_blocks(sp, rng, k):
        xb = np.ascontiguousarray(x[b * sp.batch_stride:(b + 1) * sp.batch_stride])
        yw, sw = oracle.quantize_block(xb, sp.M, sp.N, sp.row_stride, bm, bn, bi, bj)
        yg = yv[b, bi * bm:bi * bm + yw.shape[0], bj * bn:bj * bn + yw.shape[1]].cpu().numpy()
        sg = float(sv[b, bi, bj].item())
        assert np.array_equal(yg, yw), (sp.name, b, bi, bj, int((yg != yw).sum()))
        assert np.float32(sg).view(np.uint32) == np.float32(sw).view(np.uint32), (sp.name, b, bi, bj)
        n += 1
    return n


def no_nan_codes(out: Outputs) -> bool:
    return not bool(((out.y.view & 0x7F) == 0x7F).any().item())
