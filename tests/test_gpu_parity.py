"""GPU parity: every e4m3 byte and every descale bit of the CUDA library equals
the CPU oracle, on the same seeded inputs, through the C ABI.

Covers the small workload (directed blocks), the edge workload (ragged fp32
and bf16 shapes, [1,128] and [64,64] blocks, row-padded inputs), a full
Qwen3-8B-shaped layer, a full MoE layer with 128-expert stacks, misaligned
pointers, degenerate shapes, each kernel variant, canary bands around every
output, the Python conveniences, and the TMA kernel's bounded-wait error path.
"""
import numpy as np
import pytest
import torch

import blockwise_fp8_weight_b200 as fq
import oracle
from synth import TensorSpec, DIST_STUDENT_T3
from synth import workloads as W
from tests.gpu_util import Outputs, assert_same, oracle_expected, run, to_device

pytestmark = pytest.mark.gpu

PATHS = {"auto": fq.FP8BQ_PATH_AUTO, "vector": fq.FP8BQ_PATH_VECTOR,
         "tma": fq.FP8BQ_PATH_TMA, "generic": fq.FP8BQ_PATH_GENERIC}


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.init()
    yield
    torch.cuda.synchronize()
    torch.cuda.empty_cache()


class Case:
    """Host inputs, device inputs and oracle outputs of a list of specs."""

    def __init__(self, specs):
        self.specs = specs
        self.host = [W.materialize(sp) for sp in specs]
        dev = [to_device(x) for x in self.host]
        self.owners = [o for o, _ in dev]
        self.ptrs = [p for _, p in dev]
        self.want = [oracle_expected(sp, x) for sp, x in zip(specs, self.host)]

    def check(self, path, **kw):
        outs = run(self.specs, self.ptrs, path, **kw)
        for sp, o, w in zip(self.specs, outs, self.want):
            assert_same(sp, o.result(), w)


@pytest.fixture(scope="module")
def small_case():
    return Case(W.small())


@pytest.fixture(scope="module")
def edge_case():
    return Case(W.edge())


@pytest.fixture(scope="module")
def qwen_layer_case():
    return Case(W.qwen3_8b_layer(0, seed=1))


@pytest.fixture(scope="module")
def moe_layer_case():
    return Case(W.moe_layer(0))


@pytest.mark.parametrize("path", list(PATHS))
def test_small_workload(small_case, path):
    small_case.check(PATHS[path])
    y, s = small_case.want[0]
    assert s[0, 1, 0] == 1.0 and s[0, 0, 1] == np.float32(np.float32(1e-10) / np.float32(448))


@pytest.mark.parametrize("path", list(PATHS))
def test_edge_workload_one_call(edge_case, path):
    """All edge tensors (both dtypes, mixed block shapes) in one batched call."""
    edge_case.check(PATHS[path])


def test_edge_workload_one_call_per_tensor(edge_case):
    for sp, p, w in zip(edge_case.specs, edge_case.ptrs, edge_case.want):
        (o,) = run([sp], [p])
        assert_same(sp, o.result(), w)


@pytest.mark.parametrize("path", ["auto", "tma", "generic"])
def test_qwen3_8b_layer(qwen_layer_case, path):
    qwen_layer_case.check(PATHS[path])


@pytest.mark.parametrize("path", ["auto", "tma"])
def test_moe_layer(moe_layer_case, path):
    moe_layer_case.check(PATHS[path])


@pytest.mark.parametrize("dtype,xoff,yoff", [("bf16", 2, 0), ("bf16", 8, 0), ("bf16", 0, 1),
                                             ("bf16", 0, 4), ("f32", 4, 0), ("f32", 8, 2)])
def test_misaligned_pointers(dtype, xoff, yoff):
    sp = TensorSpec(f"mis.{dtype}", 300, 520, dtype=dtype, seed=61, tensor_id=xoff * 10 + yoff,
                    dist=DIST_STUDENT_T3)
    x = W.materialize(sp)
    owner, ptr = to_device(x, offset_bytes=xoff)
    want = oracle_expected(sp, x)
    for path in PATHS.values():
        (o,) = run([sp], [ptr], path, y_offsets=[yoff])
        assert_same(sp, o.result(), want)
    del owner


@pytest.mark.parametrize("dtype,M,N,ld,block,batch", [
    ("bf16", 300, 4100, None, (128, 128), 1),   # last vector of a row: upper half outside
    ("bf16", 200, 1028, 1036, (64, 64), 1),     # padded rows (poison in the padding)
    ("bf16", 37, 516, None, (1, 128), 1),       # stacked 1x128 blocks, ragged stack
    ("bf16", 130, 4100, None, (128, 128), 3),   # expert stack, 8-byte-aligned strides
    ("bf16", 129, 4100, None, (128, 128), 3),   # odd experts start 8 bytes past 16
    ("f32", 300, 4098, None, (128, 128), 1),
    ("f32", 200, 1030, 1034, (64, 64), 1),
    ("f32", 37, 514, None, (1, 128), 1),
])
def test_half_vector_rows(dtype, M, N, ld, block, batch):
    """Rows that are 8-byte but not 16-byte aligned take the vector kernel in
    8-byte halves; where a row ends inside a vector its upper half is neither
    read nor written."""
    sp = TensorSpec(f"half.{dtype}.{batch}x{M}x{N}.b{block[0]}x{block[1]}", M, N, batch=batch,
                    ld=ld, dtype=dtype, block=block, seed=73, tensor_id=M * 131 + N,
                    dist=DIST_STUDENT_T3)
    x = W.materialize(sp)
    owner, ptr = to_device(x)
    assert fq.fp8bq_path_for(Outputs(sp).desc(ptr)) == fq.FP8BQ_PATH_VECTOR
    want = oracle_expected(sp, x)
    for path in (PATHS["auto"], PATHS["vector"]):
        (o,) = run([sp], [ptr], path)
        assert_same(sp, o.result(), want)
    del owner


@pytest.mark.parametrize("shape,block", [
    ((1, 1), (128, 128)), ((5, 5), (128, 128)), ((1, 4096), (1, 128)), ((4096, 1), (128, 128)),
    ((7, 9), (1, 1)), ((256, 256), (256, 256)), ((300, 17), (64, 16)), ((130, 136), (2, 8)),
    ((64, 4096), (16, 4096)), ((33, 48), (32, 16)),
])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_degenerate_shapes_and_blocks(shape, block, dtype):
    M, N = shape
    assert block[0] * block[1] <= 65536     # the largest block the contract allows
    sp = TensorSpec(f"deg.{M}x{N}.b{block}", M, N, block=block, dtype=dtype, seed=71,
                    tensor_id=M * 7919 + N, dist=DIST_STUDENT_T3)
    x = W.materialize(sp)
    owner, ptr = to_device(x)
    want = oracle_expected(sp, x)
    for path in PATHS.values():
        (o,) = run([sp], [ptr], path)
        assert_same(sp, o.result(), want)
    del owner


@pytest.mark.parametrize("shape,block,dtype,ld", [
    ((1, 1 << 22), (1, 128), "bf16", None),        # 8 MB: folded into 256 rows
    ((1, 1 << 22), (128, 128), "bf16", None),      # one block row: blocks of 1 row, folded
    ((3, 3 << 20), (1, 128), "f32", None),         # folded by 2^k while gn allows
    ((8, 1 << 20), (128, 128), "bf16", None),      # blocks of 8 rows
    ((2, (1 << 21) + 64), (1, 64), "bf16", None),  # gn odd: no fold
    ((4, 1 << 20), (64, 128), "bf16", 1 << 20 | 64),  # padded rows: blocks of 4 rows, no fold
    ((40, 1 << 18), (128, 128), "bf16", None),     # more than a quarter block: unchanged
    ((1, 64 * 32769), (1, 4), "bf16", None),       # folded by 8, not 16: rows stay 16-byte vectors
])
def test_few_row_tensors(shape, block, dtype, ld):
    """Tensors of a few rows, which the planner runs on an equivalent geometry
    (blocks of their M rows, row-wise blocks folded into more rows): every
    code and descale against the oracle, on every path."""
    M, N = shape
    sp = TensorSpec(f"few.{M}x{N}.b{block}", M, N, block=block, dtype=dtype, ld=ld, seed=73,
                    tensor_id=M * 131 + block[0], dist=DIST_STUDENT_T3, row_lognormal_sigma=1.0)
    x = W.materialize(sp)
    owner, ptr = to_device(x)
    want = oracle_expected(sp, x)
    for path in PATHS.values():
        (o,) = run([sp], [ptr], path)
        assert_same(sp, o.result(), want)
        assert fq.fp8bq_launch_count([o.desc(ptr)]) == 1
    del owner


@pytest.mark.parametrize("shape,block,dtype,ld", [
    ((1000, 1024), (1, 128), "f32", None),     # 32-lane team, 8 stacked one-row blocks
    ((777, 1030), (1, 128), "f32", None),      # the same on rows only 8-byte aligned
    ((1000, 1024), (2, 128), "bf16", None),    # 32-lane team: two rows of 16 vectors
    ((600, 1024), (1, 256), "bf16", None),     # 32-lane team: one row of 32 vectors
    ((1000, 1024), (64, 64), "f32", None),     # 128-thread team
    ((1000, 1024), (128, 64), "bf16", 1088),   # 128-thread team, padded rows
])
def test_stacked_and_mid_size_teams(shape, block, dtype, ld):
    """Block shapes served by the 32-lane stacked-block team and the 128-thread
    team: every code and descale against the oracle, on every path."""
    M, N = shape
    sp = TensorSpec(f"team.{M}x{N}.b{block}.{dtype}", M, N, block=block, dtype=dtype, ld=ld,
                    seed=79, tensor_id=M + block[0] * 7 + block[1], dist=DIST_STUDENT_T3,
                    row_lognormal_sigma=1.0)
    x = W.materialize(sp)
    owner, ptr = to_device(x)
    want = oracle_expected(sp, x)
    for path in PATHS.values():
        (o,) = run([sp], [ptr], path)
        assert_same(sp, o.result(), want)
    del owner


def test_all_zero_and_one_element_blocks():
    sp = TensorSpec("zeros", 200, 264, seed=0)
    x = np.zeros(sp.numel_storage, dtype=np.uint16)
    x[::2] = 0x8000                                   # half the zeros are negative
    owner, ptr = to_device(x)
    want = oracle_expected(sp, x)
    for path in PATHS.values():
        (o,) = run([sp], [ptr], path)
        y, s = o.result()
        assert_same(sp, (y, s), want)
        assert set(np.unique(y)) == {0x00, 0x80}
    del owner


def test_empty_tensor_launches_nothing():
    d = fq.fp8bq_desc()
    d.M, d.N, d.ld, d.batch, d.block_m, d.block_n = 0, 128, 128, 1, 128, 128
    assert fq.fp8bq_quantize_batched([d]) == fq.FP8BQ_OK
    assert fq.fp8bq_sync_status() == fq.FP8BQ_OK


def test_non_default_stream_and_python_api():
    sp = W.qwen3_8b_layer(0, seed=5)[1]               # k_proj 1024x4096
    x = W.materialize(sp)
    want = oracle_expected(sp, x)
    xt = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).reshape(sp.M, sp.N).cuda()
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        y, d = fq.scaled_fp8_blockwise(xt, [128, 128])
    s.synchronize()
    assert y.dtype == torch.float8_e4m3fn and y.shape == (sp.M, sp.N)
    assert d.dtype == torch.float32 and d.shape == (8, 32)
    assert_same(sp, (y.view(torch.uint8).cpu().numpy()[None], d.cpu().numpy()[None]), want)
    # quant_weights: the (name, fp8), (name_scale_inv, descale) stream, one call
    out = fq.quant_weights([("a.weight", xt), ("b.weight", xt[:512])])
    assert [n for n, _ in out] == ["a.weight", "a.weight_scale_inv", "b.weight",
                                   "b.weight_scale_inv"]
    torch.cuda.synchronize()
    assert torch.equal(out[0][1].view(torch.uint8), y.view(torch.uint8))
    assert torch.equal(out[2][1].view(torch.uint8), y[:512].view(torch.uint8))
    assert torch.equal(out[3][1], d[:4])


def test_quant_weights_mixed_list_against_the_oracle():
    """quant_weights over a mixed list (bf16 and fp32, an expert stack, a
    ragged shape, a column slice with row padding): one grouped call whose
    outputs are views of two shared allocations; every byte and descale
    against the oracle, every view disjoint from the others."""
    specs = [
        TensorSpec("w.a", 1024, 4096, seed=77, tensor_id=1, row_lognormal_sigma=0.5),
        TensorSpec("w.b", 130, 129, seed=77, tensor_id=2, dist=DIST_STUDENT_T3),
        TensorSpec("w.c", 256, 384, dtype="f32", seed=77, tensor_id=3),
        TensorSpec("w.d", 512, 768, batch=4, seed=77, tensor_id=4, batch_lognormal_sigma=0.7),
        TensorSpec("w.e", 300, 200, ld=264, seed=77, tensor_id=5),
    ]
    tens, wants = [], []
    for sp in specs:
        x = W.materialize(sp)
        wants.append(oracle_expected(sp, x))
        dt = torch.bfloat16 if sp.dtype == "bf16" else torch.float32
        raw = torch.from_numpy(x.view(np.int16) if sp.dtype == "bf16" else x).view(dt).cuda()
        t = raw.reshape(sp.batch, sp.M, sp.row_stride)[..., :sp.N]
        tens.append(t if sp.batch > 1 else t[0])
    out = fq.quant_weights([(sp.name, t) for sp, t in zip(specs, tens)])
    torch.cuda.synchronize()
    assert [n for n, _ in out] == [n for sp in specs for n in (sp.name, sp.name + "_scale_inv")]
    spans = []
    for i, sp in enumerate(specs):
        y, d = out[2 * i][1], out[2 * i + 1][1]
        assert y.dtype == torch.float8_e4m3fn and y.shape == tens[i].shape and y.is_contiguous()
        gm, gn = sp.grid
        assert d.shape == ((sp.batch, gm, gn) if sp.batch > 1 else (gm, gn))
        assert_same(sp, (y.view(torch.uint8).cpu().numpy().reshape(sp.batch, sp.M, sp.N),
                         d.cpu().numpy().reshape(sp.batch, gm, gn)), wants[i])
        for t in (y, d):
            spans.append((t.data_ptr(), t.data_ptr() + t.numel() * t.element_size()))
    spans.sort()
    assert all(a[1] <= b[0] for a, b in zip(spans, spans[1:]))


def test_expert_stack_python_api():
    sp = W.moe_layer(3)[5]                             # w2 [128, 2048, 768]
    sp = TensorSpec(sp.name, sp.M, sp.N, batch=8, seed=sp.seed, tensor_id=sp.tensor_id,
                    batch_lognormal_sigma=0.7)
    x = W.materialize(sp)
    want = oracle_expected(sp, x)
    xt = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).reshape(8, sp.M, sp.N).cuda()
    y, d = fq.scaled_fp8_blockwise(xt)
    torch.cuda.synchronize()
    assert y.shape == (8, 2048, 768) and d.shape == (8, 16, 6)
    assert_same(sp, (y.view(torch.uint8).cpu().numpy(), d.cpu().numpy()), want)


def test_variant_bytes_agree_on_large_input(qwen_layer_case):
    """The vector and TMA variants write identical bytes on a full layer."""
    a = run(qwen_layer_case.specs, qwen_layer_case.ptrs, fq.FP8BQ_PATH_VECTOR)
    b = run(qwen_layer_case.specs, qwen_layer_case.ptrs, fq.FP8BQ_PATH_TMA)
    for oa, ob in zip(a, b):
        assert torch.equal(oa.y.view, ob.y.view) and torch.equal(oa.s.view, ob.s.view)


def test_tma_bounded_wait_reports_timeout_and_recovers():
    """The first CTA arms its first barrier without issuing the copy, so its
    consumers' wait can only run out: the kernel must return, report
    FP8BQ_ERR_DEVICE_TIMEOUT, and leave the context usable."""
    sp = W.qwen3_8b_layer(0, seed=9)[0]                # q_proj 4096x4096
    x = W.materialize(sp)
    owner, ptr = to_device(x)
    want = oracle_expected(sp, x)
    assert fq.fp8bq_debug_set_wait_limit_ns(5_000_000) == fq.FP8BQ_OK   # 5 ms
    assert fq.fp8bq_debug_set_inject(fq.FP8BQ_INJECT_DROP_FIRST_LOAD) == fq.FP8BQ_OK
    try:
        from tests.gpu_util import Outputs
        o = Outputs(sp)
        fq.fp8bq_set_path(fq.FP8BQ_PATH_TMA)
        assert fq.fp8bq_quantize_batched([o.desc(ptr)]) == fq.FP8BQ_OK
        assert fq.fp8bq_sync_status() == fq.FP8BQ_ERR_DEVICE_TIMEOUT
        assert fq.fp8bq_sync_status() == fq.FP8BQ_OK          # the word was cleared
        assert o.y.canaries_intact() and o.s.canaries_intact()
    finally:
        fq.fp8bq_debug_set_inject(0)
        fq.fp8bq_debug_set_wait_limit_ns(0)
        fq.fp8bq_set_path(fq.FP8BQ_PATH_AUTO)
    (o2,) = run([sp], [ptr], fq.FP8BQ_PATH_TMA)
    assert_same(sp, o2.result(), want)
    del owner


def test_grouped_call_replays_in_a_cuda_graph(qwen_layer_case):
    """The grouped call only enqueues kernels (its descriptor table travels in
    the kernel parameters), so once warmed up it can be captured in a CUDA
    graph; replays write the same bytes as the oracle."""
    from tests.gpu_util import Outputs
    case = qwen_layer_case
    outs = [Outputs(sp) for sp in case.specs]
    descs = (fq.fp8bq_desc * len(outs))(*[o.desc(p) for o, p in zip(outs, case.ptrs)])
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        assert fq.fp8bq_quantize_batched(descs, stream=s) == fq.FP8BQ_OK   # warm-up
    s.synchronize()
    for o in outs:                                   # clear the outputs before replaying
        o.y.view.fill_(0)
        o.s.view.fill_(0)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        st = fq.fp8bq_quantize_batched(descs, stream=s)
    assert st == fq.FP8BQ_OK
    g.replay()
    g.replay()
    torch.cuda.synchronize()
    assert fq.fp8bq_sync_status() == fq.FP8BQ_OK
    for sp, o, w in zip(case.specs, outs, case.want):
        assert_same(sp, o.result(), w)


@pytest.mark.parametrize("block", [(128, 128), (1, 128), (64, 64)])
@pytest.mark.parametrize("path", ["auto", "vector", "generic"])
def test_many_tensors_in_one_call(path, block):
    """700 tensors of mixed shapes in one grouped call: the list is split into
    several launches (320 descriptors per vector/generic pack, 128 per TMA
    pack), tensors of different widths share a launch, and every tensor still
    matches the oracle."""
    rng = np.random.default_rng(101)
    specs = []
    for i in range(700):
        M = int(rng.integers(1, 5)) * 128 + int(rng.integers(0, 2)) * int(rng.integers(1, 127))
        N = int(rng.choice([128, 256, 384, 1024]))
        specs.append(TensorSpec(f"many.{i}", M, N, block=block, seed=111, tensor_id=i,
                                sigma=0.02, outlier_p=1e-3))
    hosts = [W.materialize(sp) for sp in specs]
    # one device buffer for all inputs, 256-byte aligned offsets
    offs, o = [], 0
    for x in hosts:
        offs.append(o)
        o += (x.nbytes + 255) // 256 * 256
    buf = torch.empty(o, dtype=torch.uint8, device="cuda")
    for x, off in zip(hosts, offs):
        buf[off:off + x.nbytes].copy_(torch.from_numpy(x.view(np.uint8)))
    outs = run(specs, [buf.data_ptr() + off for off in offs], PATHS[path])
    for sp, x, out in zip(specs, hosts, outs):
        assert_same(sp, out.result(), oracle_expected(sp, x))


@pytest.mark.skipif(torch.cuda.device_count() < 2, reason="needs two CUDA devices")
def test_two_devices_in_one_process():
    """Kernel attributes and grid sizes are set up per device, so one process
    may quantize on one GPU, then another, then the first again."""
    specs = [TensorSpec("dev.tma", 1000, 4096, seed=81, tensor_id=1, dist=DIST_STUDENT_T3),
             TensorSpec("dev.halves", 1000, 4100, seed=81, tensor_id=2, dist=DIST_STUDENT_T3),
             TensorSpec("dev.act", 100, 4096, block=(1, 128), seed=81, tensor_id=3)]
    hosts = [W.materialize(sp) for sp in specs]
    wants = [oracle_expected(sp, x) for sp, x in zip(specs, hosts)]
    for dev in (0, 1, 0):
        with torch.cuda.device(dev):
            owners = [to_device(x) for x in hosts]
            outs = run(specs, [p for _, p in owners])
            for sp, o, w in zip(specs, outs, wants):
                assert_same(sp, o.result(), w)
            del owners, outs


def test_concurrent_groups_keep_stream_order(edge_case):
    """A call whose tensors take several kernel variants runs its launch
    groups side by side on library streams forked from the caller's stream and
    joined back: work the caller enqueues next on its stream (here a copy of
    every output, with no host synchronization in between) sees every byte."""
    from tests.gpu_util import Outputs
    case = edge_case
    outs = [Outputs(sp) for sp in case.specs]
    descs = [o.desc(p) for o, p in zip(outs, case.ptrs)]
    s = torch.cuda.Stream()
    for _ in range(3):
        for o in outs:                                   # stale bytes the copies must not see
            o.y.view.fill_(0x7F)
            o.s.view.fill_(0xFF)
        torch.cuda.synchronize()
        with torch.cuda.stream(s):
            assert fq.fp8bq_quantize_batched(descs, stream=s) == fq.FP8BQ_OK
            copies = [(o.y.view.clone(), o.s.view.clone()) for o in outs]
        s.synchronize()
        assert fq.fp8bq_sync_status(s) == fq.FP8BQ_OK
        for sp, (yc, sc), w in zip(case.specs, copies, case.want):
            gm, gn = sp.grid
            assert_same(sp, (yc.cpu().numpy().reshape(sp.batch, sp.M, sp.N),
                             sc.cpu().numpy().view(np.float32).reshape(sp.batch, gm, gn)), w)


def test_calls_from_several_host_threads(edge_case, qwen_layer_case):
    """Four host threads call the library at once, each on its own stream
    (the ctypes calls release the GIL, so the library's planning, tensor-map
    cache and launch-group fork run concurrently): every output of every
    thread is the oracle's."""
    import threading
    from tests.gpu_util import Outputs
    cases = [edge_case, qwen_layer_case, edge_case, qwen_layer_case]
    outs = [[Outputs(sp) for sp in c.specs] for c in cases]
    descs = [[o.desc(p) for o, p in zip(oo, c.ptrs)] for oo, c in zip(outs, cases)]
    streams = [torch.cuda.Stream() for _ in cases]
    errors = []
    start = threading.Barrier(len(cases))

    def work(k):
        try:
            start.wait()
            for _ in range(10):
                st = fq.fp8bq_quantize_batched(descs[k], stream=streams[k])
                assert st == fq.FP8BQ_OK, fq.fp8bq_status_string(st)
            assert fq.fp8bq_sync_status(streams[k]) == fq.FP8BQ_OK
        except BaseException as e:                       # reported below
            errors.append((k, repr(e)))

    threads = [threading.Thread(target=work, args=(k,)) for k in range(len(cases))]
    for t in threads:
        t.start()
    for t in threads:
        t.join(timeout=300)
    assert not any(t.is_alive() for t in threads)
    assert not errors, errors
    torch.cuda.synchronize()
    for c, oo in zip(cases, outs):
        for sp, o, w in zip(c.specs, oo, c.want):
            assert_same(sp, o.result(), w)


def test_mixed_variant_call_in_a_cuda_graph(edge_case):
    """Under graph capture the launch groups of a call stay on the capturing
    stream; replays write the oracle's bytes."""
    from tests.gpu_util import Outputs
    case = edge_case
    outs = [Outputs(sp) for sp in case.specs]
    descs = (fq.fp8bq_desc * len(outs))(*[o.desc(p) for o, p in zip(outs, case.ptrs)])
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        assert fq.fp8bq_quantize_batched(descs, stream=s) == fq.FP8BQ_OK   # warm-up
    s.synchronize()
    for o in outs:
        o.y.view.fill_(0)
        o.s.view.fill_(0)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        st = fq.fp8bq_quantize_batched(descs, stream=s)
    assert st == fq.FP8BQ_OK
    g.replay()
    torch.cuda.synchronize()
    assert fq.fp8bq_sync_status() == fq.FP8BQ_OK
    for sp, o, w in zip(case.specs, outs, case.want):
        assert_same(sp, o.result(), w)


def test_launch_count_follows_the_plan(qwen_layer_case):
    """fp8bq_launch_count reports the launches of a call as planned: one per
    kernel variant, dtype and block shape and per pack of descriptors (128 for
    the TMA kernel, 320 for the others), with AUTO's per-call size rule (a
    call whose TMA tensors hold less than 128 MiB of input runs them on the
    vector kernel)."""
    from tests.gpu_util import Outputs
    outs = [Outputs(sp) for sp in qwen_layer_case.specs]      # kept alive: distinct outputs
    lay = [o.desc(p) for o, p in zip(outs, qwen_layer_case.ptrs)]
    assert fq.fp8bq_launch_count(lay) == 1                     # 386 MB: one TMA launch
    one = lay[1]                                               # k_proj alone: 8 MB
    assert fq.fp8bq_path_for(one) == fq.FP8BQ_PATH_TMA        # its own choice ...
    assert fq.fp8bq_launch_count([one]) == 1                   # ... one (vector) launch
    sp = TensorSpec("count", 256, 256, seed=1)
    owner, ptr = to_device(W.materialize(sp))
    many = [Outputs(sp) for _ in range(200)]                  # 200 small tensors, 26 MB
    descs = [o.desc(ptr) for o in many]
    assert fq.fp8bq_launch_count(descs) == 1                   # one vector pack of <= 320
    assert fq.fp8bq_set_path(fq.FP8BQ_PATH_TMA) == fq.FP8BQ_OK
    try:
        assert fq.fp8bq_launch_count(descs) == 2               # TMA packs of <= 128
        assert fq.fp8bq_launch_count(descs + [lay[0]]) == 2    # q_proj joins the second pack
    finally:
        fq.fp8bq_set_path(fq.FP8BQ_PATH_AUTO)
    del owner


def test_bench_launch_counts():
    """The launch counts the benchmark reports (from the library's plan): the
    edge set takes 7 launches (bf16: TMA pairs, vector halves, vector 1x128,
    vector 64x64, generic; fp32: TMA, generic), the whole weight set 2 (TMA
    packs of 128 and 124 tensors)."""
    import bench
    specs, _ = bench.workload("edge")
    lay = bench.Layout(specs)
    assert bench.count_launches(bench.build_descs(specs, lay, 1 << 40, 1 << 41, 1 << 42)) == 7
    qwen = W.qwen3_8b_model()
    lay = bench.Layout(qwen)
    assert bench.count_launches(bench.build_descs(qwen, lay, 1 << 40, 1 << 41, 1 << 42)) == 2
