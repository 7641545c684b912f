"""GPU parity at full workload sizes: every e4m3 byte and every descale bit of
the CUDA library compared with the CPU oracle.

  * The whole Qwen3-8B-shaped weight set (36 layers x 7 linear weights,
    6.95e9 bf16 elements, 423,936 blocks) in one grouped launch -- the
    benchmarked configuration -- with the default kernel choice and with the
    vector kernel forced; the 36 per-layer launches on one stream write the
    same bytes.
  * All 48 MoE layers (q, k, v, o, 128-expert w13 and w2 stacks, 1.87 GB of
    traffic per layer), streamed layer by layer, one grouped launch each.
  * The fp32 -> e4m3fn conversion of the kernels over every fp32 bit pattern
    of magnitude <= 448, through blocks whose absmax is exactly 448 (scale 1).

The oracle is single-threaded; a pool of spawned processes runs it on many
matrices side by side (tests/oracle_pool.py), reading inputs and GPU outputs
from shared host memory.  A few sampled blocks are checked first, so that a
mismatch reports its block before the full comparison runs.
"""
import numpy as np
import pytest
import torch

import blockwise_fp8_weight_b200 as fq
import oracle
from synth import TensorSpec
from synth import workloads as W
from tests import oracle_pool as OP
from tests.gpu_util import check_sampled, no_nan_codes, run, to_device

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    yield
    torch.cuda.synchronize()
    torch.cuda.empty_cache()


@pytest.fixture(scope="module")
def pool():
    p = OP.make_pool()
    yield p
    p.close()


def align(v: int, a: int = 256) -> int:
    return (v + a - 1) // a * a


def offsets(sizes) -> tuple[list[int], int]:
    out, o = [], 0
    for n in sizes:
        out.append(o)
        o = align(o + n)
    return out, o


class HostSet:
    """Inputs of a tensor list packed into one shared host buffer (256-byte
    aligned offsets), and room for the GPU's codes and descales."""

    def __init__(self, specs, tag: str):
        self.specs = specs
        self.x_off, xb = offsets(sp.numel_storage * sp.elem_bytes for sp in specs)
        self.y_off, yb = offsets(sp.numel for sp in specs)
        self.s_off, sb = offsets(sp.nblocks * 4 for sp in specs)
        self.x = OP.ShmBuffer(xb, tag + "_x")
        self.y = OP.ShmBuffer(yb, tag + "_y")
        self.s = OP.ShmBuffer(sb, tag + "_s")

    def generate(self, specs=None) -> None:
        self.specs = specs or self.specs
        for sp, o in zip(self.specs, self.x_off):
            W.materialize_into(sp, self.x.ptr + o)

    def host_x(self, i: int) -> np.ndarray:
        sp = self.specs[i]
        n = sp.numel_storage * sp.elem_bytes
        return self.x.mm[self.x_off[i]:self.x_off[i] + n].view(sp.np_dtype)

    def collect(self, outs) -> None:
        """Copy every output (codes, descales) into the shared buffers."""
        for o, yo, so in zip(outs, self.y_off, self.s_off):
            torch.from_numpy(self.y.mm[yo:yo + o.y.nbytes]).copy_(o.y.view)
            torch.from_numpy(self.s.mm[so:so + o.s.nbytes]).copy_(o.s.view)
        self.y.mm.flush()
        self.s.mm.flush()

    def tasks(self):
        return OP.tasks_for(self.specs, self.x.path, self.x_off, self.y.path, self.y_off,
                            self.s.path, self.s_off)

    def close(self) -> None:
        for b in (self.x, self.y, self.s):
            b.close()


def assert_all_equal(results, want_matrices: int) -> None:
    n, errs = OP.summarize(results)
    assert not errs, "\n".join(errs[:20])
    assert n == want_matrices, (n, want_matrices)


@pytest.fixture(scope="module")
def whole_model():
    specs = W.qwen3_8b_model()
    hs = HostSet(specs, "model")
    try:
        hs.generate()
        dev = torch.empty(hs.x.nbytes, dtype=torch.uint8, device="cuda")
        dev.copy_(torch.from_numpy(hs.x.mm))
        ptrs = [dev.data_ptr() + o for o in hs.x_off]
        yield hs, ptrs
        del dev
        torch.cuda.empty_cache()
    finally:
        hs.close()


def test_whole_model_one_grouped_launch(whole_model, pool):
    """Config: the whole weight set, one call; every block against the oracle."""
    hs, ptrs = whole_model
    specs = hs.specs
    outs = run(specs, ptrs)                    # one call, 252 tensors
    rng = np.random.default_rng(2024)
    assert sum(check_sampled(sp, hs.host_x(i), o, rng, k=2)
               for i, (sp, o) in enumerate(zip(specs, outs))) >= 252 * 4
    for o in outs:
        assert o.y.canaries_intact() and o.s.canaries_intact()
        assert no_nan_codes(o)
    hs.collect(outs)
    pending = pool.map_async(OP.verify, hs.tasks())
    # meanwhile: the per-layer streamed form writes the same bytes
    for layer in range(W.QWEN3_8B_LAYERS):
        sl = slice(7 * layer, 7 * layer + 7)
        per = run(specs[sl], ptrs[sl])
        for a, b in zip(per, outs[sl]):
            assert torch.equal(a.y.view, b.y.view) and torch.equal(a.s.view, b.s.view)
        del per
    assert_all_equal(pending.get(), 252)


def test_whole_model_vector_variant(whole_model, pool):
    """The same call with the vector kernel forced, every block against the oracle."""
    hs, ptrs = whole_model
    outs = run(hs.specs, ptrs, fq.FP8BQ_PATH_VECTOR)
    for o in outs:
        assert o.y.canaries_intact() and o.s.canaries_intact()
    hs.collect(outs)
    del outs
    assert_all_equal(pool.map(OP.verify, hs.tasks()), 252)


def test_moe_layers_streamed(pool):
    """All 48 MoE layers, one grouped launch per layer on one stream; every
    expert matrix of every layer against the oracle.  Host buffers rotate
    between two sets, so layer l + 1 is generated while layer l is checked."""
    sets = [HostSet(W.moe_layer(0), f"moe{k}") for k in range(2)]
    xdev = torch.empty(sets[0].x.nbytes, dtype=torch.uint8, device="cuda")
    pending = [None, None]
    results = []
    rng = np.random.default_rng(5)
    try:
        for layer in range(W.MOE_LAYERS):
            k = layer % 2
            hs = sets[k]
            if pending[k] is not None:
                results += pending[k].get()
                pending[k] = None
            hs.generate(W.moe_layer(layer))
            xdev.copy_(torch.from_numpy(hs.x.mm))
            ptrs = [xdev.data_ptr() + o for o in hs.x_off]
            outs = run(hs.specs, ptrs)
            for i, (sp, o) in enumerate(zip(hs.specs, outs)):
                assert o.y.canaries_intact() and o.s.canaries_intact(), sp.name
                if layer in (0, W.MOE_LAYERS - 1):
                    check_sampled(sp, hs.host_x(i), o, rng, k=2)
            hs.collect(outs)
            del outs
            pending[k] = pool.map_async(OP.verify, hs.tasks())
        for p in pending:
            if p is not None:
                results += p.get()
    finally:
        for hs in sets:
            hs.close()
        del xdev
        torch.cuda.empty_cache()
    # 4 plain matrices + 2 x 128 experts per layer
    assert_all_equal(results, W.MOE_LAYERS * (4 + 2 * 128))


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
