"""GPU parity of the dequantization kernels (decode(y) * descale, fp32
product rounded to nearest even, then to bf16 for bf16 output) against the
oracle, bit for bit, through the C ABI; codes and descales come from the
oracle's quantization of seeded inputs."""
import numpy as np
import pytest
import torch

import blockwise_fp8_weight_b200 as fq
import oracle
from synth import DIST_STUDENT_T3, TensorSpec
from synth import workloads as W
from tests.gpu_util import Guarded

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    yield
    torch.cuda.synchronize()


def run_dequant(y, s, M, N, bm, bn, out_dtype, batch=1, ld_out=None, path=fq.FP8BQ_PATH_AUTO,
                y_offset=0):
    ld_out = N if ld_out is None else ld_out
    oes = 2 if out_dtype == "bf16" else 4
    obs = (M - 1) * ld_out + N + 8 if batch > 1 else 0
    yt = torch.empty(y.size + y_offset, dtype=torch.uint8, device="cuda")
    yt[y_offset:].copy_(torch.from_numpy(y.reshape(-1)))
    st = torch.from_numpy(s.reshape(-1).copy()).cuda()
    span = (batch - 1) * obs + (M - 1) * ld_out + N
    out = Guarded(span * oes)
    fq.fp8bq_set_path(path)
    try:
        status = fq.fp8bq_dequantize(yt.data_ptr() + y_offset, st, batch, M, N, bm, bn, out.ptr,
                                     fq.FP8BQ_BF16 if oes == 2 else fq.FP8BQ_F32, ld_out, obs)
    finally:
        fq.fp8bq_set_path(fq.FP8BQ_PATH_AUTO)
    assert status == fq.FP8BQ_OK, fq.fp8bq_status_string(status)
    assert fq.fp8bq_sync_status() == fq.FP8BQ_OK
    assert out.canaries_intact()
    raw = out.numpy().view(np.uint16 if oes == 2 else np.float32)
    res = np.empty((batch, M, N), dtype=raw.dtype)
    for b in range(batch):
        for r in range(M):
            o = b * obs + r * ld_out
            res[b, r] = raw[o:o + N]
    return res


def expected(y, s, bm, bn, out_dtype):
    return np.stack([oracle.dequantize(y[b], s[b], bm, bn, out_dtype) for b in range(y.shape[0])])


def quantized(sp):
    x = W.materialize(sp)
    ys, ss = [], []
    for b in range(sp.batch):
        xb = np.ascontiguousarray(x[b * sp.batch_stride:(b + 1) * sp.batch_stride])
        yb, sb = oracle.quantize(xb, sp.M, sp.N, sp.row_stride, *sp.block)
        ys.append(yb)
        ss.append(sb)
    return np.stack(ys), np.stack(ss)


CASES = [
    TensorSpec("q", 1024, 4096, seed=81, tensor_id=1, sigma=0.02, row_lognormal_sigma=0.5,
               outlier_p=1e-3),
    TensorSpec("ragged", 130, 129, seed=81, tensor_id=2, dist=DIST_STUDENT_T3),
    TensorSpec("f32src", 300, 520, dtype="f32", seed=81, tensor_id=3, dist=DIST_STUDENT_T3),
    TensorSpec("b1x128", 64, 4096, block=(1, 128), seed=81, tensor_id=4, sigma=1.0,
               row_lognormal_sigma=1.0),
    TensorSpec("b64", 200, 192, block=(64, 64), seed=81, tensor_id=5),
    TensorSpec("experts", 256, 768, batch=4, seed=81, tensor_id=6, batch_lognormal_sigma=0.7),
    TensorSpec("odd_block", 100, 96, block=(5, 48), seed=81, tensor_id=7),
    TensorSpec("tile_edges", 130, 400, block=(32, 16), seed=81, tensor_id=8),  # ragged tiles
]


@pytest.mark.parametrize("sp", CASES, ids=[c.name for c in CASES])
@pytest.mark.parametrize("out_dtype", ["bf16", "f32"])
@pytest.mark.parametrize("path", ["auto", "vector", "generic"])
def test_dequantize_matches_oracle(sp, out_dtype, path):
    """Every kernel: AUTO (the vector kernel where rows and blocks allow it),
    VECTOR forced, GENERIC forced."""
    y, s = quantized(sp)
    want = expected(y, s, *sp.block, out_dtype)
    P = {"auto": fq.FP8BQ_PATH_AUTO, "vector": fq.FP8BQ_PATH_VECTOR,
         "generic": fq.FP8BQ_PATH_GENERIC}[path]
    got = run_dequant(y, s, sp.M, sp.N, *sp.block, out_dtype, batch=sp.batch, path=P)
    assert np.array_equal(got.view(np.uint32 if out_dtype == "f32" else np.uint16),
                          want.view(np.uint32 if out_dtype == "f32" else np.uint16))
    got2 = run_dequant(y, s, sp.M, sp.N, *sp.block, out_dtype, batch=sp.batch,
                       ld_out=sp.N + 24, path=P, y_offset=3)
    assert np.array_equal(got2.view(got.dtype), got)


def test_dequantize_every_code_and_scale():
    """All 256 codes (NaN codes included) against many scales: powers of two,
    1, random fp32 values from 1e-30 to 1e30."""
    rng = np.random.default_rng(3)
    scales = np.concatenate([2.0 ** np.arange(-40, 41, 3), [1.0],
                             10.0 ** rng.uniform(-30, 30, size=80)]).astype(np.float32)
    M, N = len(scales), 256
    y = np.tile(np.arange(256, dtype=np.uint8), (M, 1))
    s = scales.reshape(M, 1)
    for out_dtype in ("bf16", "f32"):
        want = oracle.dequantize(y, s, 1, 256, out_dtype)
        got = run_dequant(y[None], s[None], M, N, 1, 256, out_dtype)[0]
        if out_dtype == "f32":
            nan = np.isnan(want)
            assert np.array_equal(np.isnan(got), nan)
            assert nan.sum() == 2 * M                     # codes 0x7F and 0xFF
            assert np.array_equal(got.view(np.uint32)[~nan], want.view(np.uint32)[~nan])
        else:
            def is_nan(h):
                return ((h & 0x7F80) == 0x7F80) & ((h & 0x7F) != 0)
            nan = is_nan(want)
            assert np.array_equal(is_nan(got), nan)
            assert np.array_equal(got[~nan], want[~nan])


def test_roundtrip_python_api():
    sp = W.qwen3_8b_layer(0, seed=5)[1]
    x = W.materialize(sp)
    xt = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).reshape(sp.M, sp.N).cuda()
    y, d = fq.scaled_fp8_blockwise(xt)
    back = fq.dequantize_fp8_blockwise(y, d)
    back32 = fq.dequantize_fp8_blockwise(y, d, out_dtype=torch.float32)
    torch.cuda.synchronize()
    yo, so = oracle.quantize(x, sp.M, sp.N)
    assert np.array_equal(back.view(torch.int16).cpu().numpy().view(np.uint16),
                          oracle.dequantize(yo, so, 128, 128, "bf16"))
    assert np.array_equal(back32.cpu().numpy(), oracle.dequantize(yo, so, 128, 128, "f32"))


def test_dequantize_batched_mixed_list():
    """One grouped call over stacks that take different kernels (vector and
    element-wise) and output dtypes equals the oracle on every element."""
    specs = [CASES[0], CASES[1], CASES[3], CASES[5], CASES[6]]
    dtypes = ["bf16", "f32", "bf16", "bf16", "f32"]
    descs, outs, wants = [], [], []
    keep = []
    for sp, od in zip(specs, dtypes):
        y, s = quantized(sp)
        wants.append(expected(y, s, *sp.block, od))
        yt = torch.from_numpy(y.reshape(-1).copy()).cuda()
        st = torch.from_numpy(s.reshape(-1).copy()).cuda()
        oes = 2 if od == "bf16" else 4
        out = Guarded(sp.batch * sp.M * sp.N * oes)
        keep += [yt, st]
        outs.append(out)
        d = fq.fp8bq_dequant_desc()
        d.y_u8, d.descale_f32, d.out = yt.data_ptr(), st.data_ptr(), out.ptr
        d.batch, d.M, d.N = sp.batch, sp.M, sp.N
        d.ld_out, d.out_batch_stride = sp.N, sp.M * sp.N
        d.dtype_out = fq.FP8BQ_BF16 if od == "bf16" else fq.FP8BQ_F32
        d.block_m, d.block_n = sp.block
        d.reserved = 0
        descs.append(d)
    assert fq.fp8bq_dequantize_batched(descs) == fq.FP8BQ_OK
    assert fq.fp8bq_sync_status() == fq.FP8BQ_OK
    for sp, od, out, want in zip(specs, dtypes, outs, wants):
        assert out.canaries_intact()
        got = out.numpy().view(np.uint16 if od == "bf16" else np.uint32)
        assert np.array_equal(got, want.view(got.dtype).reshape(-1)), sp.name
