"""GPU parity at full workload sizes, on sampled blocks the oracle computes
one by one, plus properties that hold at any size.

  * The whole Qwen3-8B-shaped weight set (36 layers x 7 linear weights,
    6.95e9 bf16 elements) in one grouped launch -- the benchmarked
    configuration -- and as 36 per-layer launches on one stream.
  * MoE layers (q, k, v, o, 128-expert w13 and w2 stacks) streamed layer by
    layer.
  * The fp32 -> e4m3fn conversion of the kernels over every fp32 bit pattern
    of magnitude <= 448, through blocks whose absmax is exactly 448 (scale 1).
"""
import numpy as np
import pytest
import torch

import blockwise_fp8_weight_b200 as fq
import oracle
from synth import TensorSpec
from synth import workloads as W
from tests.gpu_util import Outputs, run, to_device

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    yield
    torch.cuda.synchronize()
    torch.cuda.empty_cache()


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
        xb = x[b * sp.batch_stride:(b + 1) * sp.batch_stride]
        yw, sw = oracle.quantize_block(xb, sp.M, sp.N, sp.row_stride, bm, bn, bi, bj)
        yg = yv[b, bi * bm:bi * bm + yw.shape[0], bj * bn:bj * bn + yw.shape[1]].cpu().numpy()
        sg = float(sv[b, bi, bj].item())
        assert np.array_equal(yg, yw), (sp.name, b, bi, bj, int((yg != yw).sum()))
        assert np.float32(sg).view(np.uint32) == np.float32(sw).view(np.uint32), (sp.name, b, bi, bj)
        n += 1
    return n


def no_nan_codes(out: Outputs) -> bool:
    return not bool(((out.y.view & 0x7F) == 0x7F).any().item())


@pytest.fixture(scope="module")
def whole_model():
    specs = W.qwen3_8b_model()
    host = [W.materialize(sp) for sp in specs]
    dev = [to_device(x) for x in host]
    yield specs, host, [p for _, p in dev]
    del dev
    torch.cuda.empty_cache()


def test_whole_model_one_grouped_launch(whole_model):
    specs, host, ptrs = whole_model
    outs = run(specs, ptrs)                    # one call, 252 tensors
    rng = np.random.default_rng(2024)
    checked = sum(check_sampled(sp, x, o, rng) for sp, x, o in zip(specs, host, outs))
    assert checked >= 252 * 4
    for o in outs:
        assert o.y.canaries_intact() and o.s.canaries_intact()
        assert no_nan_codes(o)
    # the per-layer streamed form writes the same bytes
    for layer in range(W.QWEN3_8B_LAYERS):
        sl = slice(7 * layer, 7 * layer + 7)
        per = run(specs[sl], ptrs[sl])
        for a, b in zip(per, outs[sl]):
            assert torch.equal(a.y.view, b.y.view) and torch.equal(a.s.view, b.s.view)
        del per


def test_whole_model_tma_variant(whole_model):
    specs, host, ptrs = whole_model
    outs = run(specs, ptrs, fq.FP8BQ_PATH_TMA)
    rng = np.random.default_rng(77)
    for sp, x, o in zip(specs, host, outs):
        check_sampled(sp, x, o, rng, k=3)
        assert no_nan_codes(o)


def test_moe_layers_streamed():
    rng = np.random.default_rng(5)
    layers = [0, 1, 46, 47]
    specs = [sp for l in layers for sp in W.moe_layer(l)]
    host = [W.materialize(sp) for sp in specs]
    dev = [to_device(x) for x in host]
    ptrs = [p for _, p in dev]
    outs = []
    for i in range(len(layers)):              # one grouped launch per layer, one stream
        outs += run(specs[6 * i:6 * i + 6], ptrs[6 * i:6 * i + 6])
    for sp, x, o in zip(specs, host, outs):
        check_sampled(sp, x, o, rng, k=8)
        assert no_nan_codes(o)
    del dev


@pytest.mark.parametrize("path,stride", [("auto", 1), ("tma", 13), ("generic", 29)])
def test_conversion_over_all_fp32_patterns(path, stride):
    """Rows of [448, v_1 .. v_127] with block [1, 128]: scale 1, reciprocal 1,
    so the kernel's codes are its e4m3fn conversion of every v (both signs,
    every fp32 pattern with |v| <= 448; a stride > 1 takes every stride-th)."""
    top = 0x43E00000                            # bits of 448.0
    per_chunk = 127 * (1 << 20)
    P = {"auto": fq.FP8BQ_PATH_AUTO, "tma": fq.FP8BQ_PATH_TMA, "generic": fq.FP8BQ_PATH_GENERIC}
    for sign in (0, 0x80000000):
        start = 0
        while start <= top:
            pats = np.arange(start, min(top + 1, start + per_chunk * stride), stride,
                             dtype=np.uint64).astype(np.uint32)
            start += per_chunk * stride
            rows = -(-pats.size // 127)
            vals = np.full(rows * 127, 0, dtype=np.uint32)
            vals[:pats.size] = pats | np.uint32(sign)
            x = np.empty((rows, 128), dtype=np.float32)
            x[:, 0] = 448.0
            x[:, 1:] = vals.view(np.float32).reshape(rows, 127)
            sp = TensorSpec("cvt", rows, 128, block=(1, 128), dtype="f32")
            owner, ptr = to_device(x.reshape(-1))
            (o,) = run([sp], [ptr], P[path])
            y, s = o.result()
            assert (s == 1.0).all()
            want = oracle.e4m3(x[:, 1:].reshape(-1)).reshape(rows, 127)
            got = y[0][:, 1:]
            bad = np.flatnonzero(got != want)
            assert bad.size == 0, (path, hex(int(x[:, 1:].reshape(-1)[bad[0]].view(np.uint32))),
                                   int(got.reshape(-1)[bad[0]]), int(want.reshape(-1)[bad[0]]))
            assert (y[0][:, 0] == 0x7E).all()
            del owner, o
