"""The full-size parity harness (tests/oracle_pool.py) on the CPU: tasks built
from packed shared buffers find every matrix, a spawned pool reports no
difference for outputs equal to the oracle's, and it does report a single
flipped code or descale bit at the right place."""
import numpy as np

from synth import TensorSpec, DIST_STUDENT_T3
from synth import workloads as W
from tests import oracle_pool as OP
import oracle


def _setup():
    specs = [
        TensorSpec("a", 130, 129, dtype="f32", seed=9, tensor_id=1, dist=DIST_STUDENT_T3),
        TensorSpec("stack", 70, 96, batch=5, block=(32, 64), seed=9, tensor_id=2,
                   batch_lognormal_sigma=0.7),
        TensorSpec("padded", 40, 300, ld=320, seed=9, tensor_id=3),
    ]
    def offs(sizes):
        out, o = [], 0
        for n in sizes:
            out.append(o)
            o = (o + n + 255) // 256 * 256
        return out, o
    xo, xb = offs(sp.numel_storage * sp.elem_bytes for sp in specs)
    yo, yb = offs(sp.numel for sp in specs)
    so, sb = offs(sp.nblocks * 4 for sp in specs)
    bufs = [OP.ShmBuffer(xb, "x"), OP.ShmBuffer(yb, "y"), OP.ShmBuffer(sb, "s")]
    x, y, s = bufs
    for i, sp in enumerate(specs):
        W.materialize_into(sp, x.ptr + xo[i])
        xa = x.mm[xo[i]:xo[i] + sp.numel_storage * sp.elem_bytes].view(sp.np_dtype)
        gm, gn = sp.grid
        for b in range(sp.batch):
            xm = np.ascontiguousarray(xa[b * sp.batch_stride:(b + 1) * sp.batch_stride])
            yw, sw = oracle.quantize(xm, sp.M, sp.N, sp.row_stride, *sp.block)
            y.mm[yo[i] + b * sp.M * sp.N:yo[i] + (b + 1) * sp.M * sp.N] = yw.reshape(-1)
            s.mm[so[i] + b * gm * gn * 4:so[i] + (b + 1) * gm * gn * 4] = \
                sw.reshape(-1).view(np.uint8)
    tasks = OP.tasks_for(specs, x.path, xo, y.path, yo, s.path, so, experts_per_task=2)
    return specs, bufs, (xo, yo, so), tasks


def test_pool_finds_every_matrix_and_every_difference():
    specs, bufs, (xo, yo, so), tasks = _setup()
    x, y, s = bufs
    pool = OP.make_pool(2)
    try:
        assert len(tasks) == 1 + 3 + 1          # the stack of 5 in runs of 2
        n, errs = OP.summarize(pool.map(OP.verify, tasks))
        assert (n, errs) == (1 + 5 + 1, [])
        # one flipped code in expert 3 of the stack, row 7, column 90
        sp = specs[1]
        at = yo[1] + 3 * sp.M * sp.N + 7 * sp.N + 90
        y.mm[at] ^= 0x01
        y.mm.flush()
        n, errs = OP.summarize(pool.map(OP.verify, tasks))
        assert n == 7 and len(errs) == 1
        assert errs[0].startswith("stack: 1 codes and 0 descales differ")
        assert "matrix 3 element (7, 90)" in errs[0]
        y.mm[at] ^= 0x01
        # one flipped descale bit of the padded matrix (1 x 3 blocks), block (0, 2)
        gm, gn = specs[2].grid
        assert (gm, gn) == (1, 3)
        at = so[2] + 2 * 4
        s.mm[at] ^= 0x01
        s.mm.flush()
        y.mm.flush()
        n, errs = OP.summarize(pool.map(OP.verify, tasks))
        assert len(errs) == 1 and "padded: 0 codes and 1 descales differ" in errs[0]
        assert "descale (0, 2)" in errs[0]
    finally:
        pool.close()
        for b in bufs:
            b.close()
