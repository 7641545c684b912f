"""Pins for the CPU oracle: checks against facts fixed outside the oracle.

Nothing here compares the oracle with itself.  The facts come from the
float8_e4m3fn format (an independent grid-search rounding reference and two
library casts), from closed forms of the method's steps (verl docs page
"fp8_kernel.py -- FP8 量化内核", section 2 "Triton 实现": absmax with eps
floor, scale = absmax / 448, y = clamp(x * (1 / scale)), fp8 store, scale
store), from hand-derived worked examples (tests/golden), from exact rational
arithmetic, from invariants of the definition, and from a second, naive
quantizer on small shapes.
"""
import ctypes
import json
import os
from fractions import Fraction

import ml_dtypes
import numpy as np
import pytest
import torch

import oracle
from synth import DIST_STUDENT_T3, TensorSpec, bf16_bits_to_f32, f32_to_bf16_bits
from synth import workloads as W
from tests.exact import frac, round_f32
from tests.pins import helper as H

EPS = oracle.EPS
GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "directed_blocks.json")


def as_f32(x: np.ndarray) -> np.ndarray:
    return bf16_bits_to_f32(x) if x.dtype == np.uint16 else x


# ---------------------------------------------------------------- converter


def test_converter_exhaustive_against_grid_search():
    """Every fp32 pattern with finite magnitude (and +-inf), both signs, rounds
    to the nearest e4m3fn grid value, ties to the even code, saturating."""
    addr = ctypes.cast(oracle.lib().fp8bq_oracle_e4m3, ctypes.c_void_p).value
    bad, first = H.sweep(addr, os.cpu_count() or 1)
    assert bad == 0, f"{bad} mismatches; first pattern/got/want = {[hex(v) for v in first]}"


def test_converter_matches_library_casts():
    """On a sample of clamped fp32 values, the converter equals the
    float8_e4m3fn casts of ml_dtypes and of torch (both round to nearest even)."""
    rng = np.random.default_rng(7)
    pats = rng.integers(0, 2**32, size=1 << 21, dtype=np.uint64).astype(np.uint32)
    v = pats.view(np.float32)
    # dense coverage around every grid value and midpoint, where rounding decides
    g = H.grid()
    pts = np.concatenate([g, (g[:-1] + g[1:]) / 2]).astype(np.float32)
    near = (pts.view(np.uint32)[:, None].astype(np.int64) + np.arange(-64, 65)[None, :])
    near = near[(near >= 0) & (near < 0x7F800000)].astype(np.uint32).view(np.float32)
    v = np.concatenate([v, near, -near])
    v = v[np.isfinite(v)]
    v = np.clip(v, -448.0, 448.0).astype(np.float32)
    got = oracle.e4m3(v)
    want_ml = v.astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    want_t = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(got, want_ml)
    assert np.array_equal(got, want_t)


def test_decode_matches_format_grid():
    codes = np.arange(256, dtype=np.uint8)
    d = oracle.e4m3_decode(codes).astype(np.float64)
    g = H.grid()
    assert np.array_equal(d[:127], g)
    assert np.array_equal(d[128:255], -g)
    assert np.signbit(d[128]) and d[128] == 0.0
    assert np.isnan(d[127]) and np.isnan(d[255])
    ml = codes.view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    ok = ~np.isnan(ml)
    assert np.array_equal(d[ok], ml[ok])
    assert g[126] == 448.0 and g[1] == 2.0**-9 and g[8] == 2.0**-6


# ------------------------------------------------------- worked examples


def _golden_input(values, dtype):
    x = np.array([float.fromhex(v) for v in values], dtype=np.float32)
    return f32_to_bf16_bits(x) if dtype == "bf16" else x


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_golden_directed_blocks(dtype):
    cases = json.load(open(GOLDEN))["cases"]
    for c in cases:
        bm, bn = c["block"]
        x = _golden_input(c["x"], dtype)
        assert np.array_equal(as_f32(x).astype(np.float64), [float.fromhex(v) for v in c["x"]])
        y, s = oracle.quantize(x, bm, bn, bm=bm, bn=bn)
        want = np.array([int(v, 16) for v in c["y"]], dtype=np.uint8).reshape(bm, bn)
        assert np.array_equal(y, want), (c["name"], [hex(v) for v in y.ravel()])
        if c.get("s_bits_is_eps_over_448"):
            assert frac(s[0, 0]) == round_f32(frac(EPS) / 448)
            assert int(EPS.view(np.uint32)) == 0x2EDBE6FF
        else:
            assert int(s.view(np.uint32)[0, 0]) == int(c["s_bits"], 16), c["name"]


# ------------------------------------------------------- directed blocks


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("neg", [False, True])
def test_all_zero_block(dtype, neg):
    """absmax 0 -> eps floor: scale = eps/448 correctly rounded, every byte 0
    (or 0x80 for -0)."""
    M, N = 128, 128
    if dtype == "bf16":
        x = np.full(M * N, 0x8000 if neg else 0, dtype=np.uint16)
    else:
        x = np.full(M * N, -0.0 if neg else 0.0, dtype=np.float32)
    y, s = oracle.quantize(x, M, N)
    assert s.shape == (1, 1)
    assert frac(s[0, 0]) == round_f32(frac(EPS) / 448)
    assert (y == (0x80 if neg else 0x00)).all()


def _grid_block(dtype, rng):
    """A 128x128 block holding every finite e4m3fn value (both signs, +-0),
    every midpoint between neighbours (both signs), 448 itself, and random
    grid values; with the expected code of each element, derived from the
    grid index (ties at midpoints go to the even code)."""
    g = H.grid()
    vals, codes = [], []
    for c in range(127):
        vals += [g[c], -g[c]]
        codes += [c, c | 0x80]
    for c in range(126):
        m = (g[c] + g[c + 1]) / 2
        even = c if c % 2 == 0 else c + 1
        vals += [m, -m]
        codes += [even, even | 0x80]
    rest = 128 * 128 - len(vals)
    rc = rng.integers(0, 127, size=rest)
    rs = rng.integers(0, 2, size=rest)
    vals += list(np.where(rs == 1, -g[rc], g[rc]))
    codes += list(rc | (rs << 7))
    perm = rng.permutation(len(vals))
    v = np.array(vals, dtype=np.float64)[perm]
    q = np.array(codes, dtype=np.uint8)[perm]
    x32 = v.astype(np.float32)
    assert np.array_equal(x32.astype(np.float64), v)
    if dtype == "bf16":
        x = f32_to_bf16_bits(x32)
        assert np.array_equal(bf16_bits_to_f32(x), x32)
    else:
        x = x32
    return x, q


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_absmax_448_reproduces_grid(dtype):
    """absmax exactly 448 -> scale 1, reciprocal 1: on-grid inputs come back
    bit for bit, midpoints go to the even neighbour, signs (and -0) survive."""
    x, q = _grid_block(dtype, np.random.default_rng(3))
    y, s = oracle.quantize(x, 128, 128)
    assert s[0, 0] == np.float32(1.0)
    assert np.array_equal(y.ravel(), q)


# ------------------------------------------------------- random blocks


def _random_cases():
    rng_specs = [
        TensorSpec("qwen_like", 384, 512, seed=11, tensor_id=1, sigma=0.02,
                   row_lognormal_sigma=0.5, outlier_p=1e-3),
        TensorSpec("t3_f32", 260, 390, dtype="f32", seed=12, tensor_id=2,
                   dist=DIST_STUDENT_T3, sigma=0.02),
        TensorSpec("wide_range", 256, 256, seed=13, tensor_id=3, sigma=1.0,
                   row_lognormal_sigma=3.0),
    ]
    return [(sp, W.materialize(sp)) for sp in rng_specs]


@pytest.fixture(scope="module")
def random_cases():
    return _random_cases()


def test_codes_in_range_and_argmax_saturates(random_cases):
    """No NaN code is ever produced, |dec(q)| <= 448, and in every block the
    element(s) of largest magnitude map to +-448 (0x7E / 0xFE)."""
    for sp, x in random_cases:
        y, s = oracle.quantize(x, sp.M, sp.N)
        assert not np.isin(y, [0x7F, 0xFF]).any()
        assert np.abs(oracle.e4m3_decode(y)).max() <= 448.0
        xf = as_f32(x).reshape(sp.M, sp.N)
        gm, gn = sp.grid
        for bi in range(gm):
            for bj in range(gn):
                blk = np.abs(xf[bi * 128:(bi + 1) * 128, bj * 128:(bj + 1) * 128])
                yb = y[bi * 128:(bi + 1) * 128, bj * 128:(bj + 1) * 128]
                top = blk == blk.max()
                assert blk.max() > EPS
                assert np.isin(yb[top], [0x7E, 0xFE]).all(), (sp.name, bi, bj)


def _ulp_e4m3(v: np.ndarray) -> np.ndarray:
    a = np.abs(v.astype(np.float64))
    _, e = np.frexp(a)                     # a = m * 2^e, m in [0.5, 1)
    ulp = np.ldexp(1.0, e - 1 - 3)
    return np.where(a < 2.0**-6, 2.0**-9, ulp)


def test_rounding_error_within_half_ulp(random_cases):
    """|dec(q) - v| <= ulp_e4m3(v) / 2, with v = clamp(x * r, -448, 448)."""
    for sp, x in random_cases:
        y, s = oracle.quantize(x, sp.M, sp.N)
        xf = as_f32(x).reshape(sp.M, sp.N)
        r = (np.float32(1.0) / s).astype(np.float32)
        rr = np.repeat(np.repeat(r, 128, 0), 128, 1)[:sp.M, :sp.N]
        v = np.clip(xf * rr, -448, 448).astype(np.float32)
        err = np.abs(oracle.e4m3_decode(y).astype(np.float64) - v.astype(np.float64))
        assert (err <= _ulp_e4m3(v) / 2).all()


def test_steps_round_exactly_once_each(random_cases):
    """Each step is one IEEE binary32 round-to-nearest operation, checked in
    exact rational arithmetic: scale = RN(absmax / 448), r = RN(1 / scale),
    v = RN(x * r) (no fused multiply), then nearest e4m3fn."""
    rng = np.random.default_rng(5)
    for sp, x in random_cases:
        y, s = oracle.quantize(x, sp.M, sp.N)
        xf = as_f32(x).reshape(sp.M, sp.N)
        gm, gn = sp.grid
        for bi in range(gm):
            for bj in range(gn):
                blk = xf[bi * 128:(bi + 1) * 128, bj * 128:(bj + 1) * 128]
                a = max(Fraction(float(np.abs(blk).max())), frac(EPS))
                sc = round_f32(a / 448)
                assert frac(s[bi, bj]) == sc
                rcp = round_f32(1 / sc)
                idx = rng.integers(0, blk.size, size=64)
                vs = []
                for k in idx:
                    v = round_f32(frac(blk.flat[k]) * rcp)
                    v = min(max(v, Fraction(-448)), Fraction(448))
                    vs.append(float(v))
                want = H.nearest_codes(np.array(vs))
                got = y[bi * 128:(bi + 1) * 128, bj * 128:(bj + 1) * 128].ravel()[idx]
                assert np.array_equal(got, want), (sp.name, bi, bj)


# ------------------------------------------------------- invariants


def test_power_of_two_scaling_invariance():
    """x -> x * 2^k (exact, far from under/overflow and from eps) gives
    scale * 2^k and identical codes."""
    sp = TensorSpec("p2", 256, 384, seed=21, tensor_id=0, sigma=0.02, row_lognormal_sigma=0.5)
    x = W.materialize(sp)
    xf = bf16_bits_to_f32(x)
    y0, s0 = oracle.quantize(x, sp.M, sp.N)
    for k in (-7, -1, 3, 9):
        xk = f32_to_bf16_bits(xf * np.float32(2.0**k))
        assert np.array_equal(bf16_bits_to_f32(xk), xf * np.float32(2.0**k))
        yk, sk = oracle.quantize(xk, sp.M, sp.N)
        assert np.array_equal(yk, y0)
        assert np.array_equal(sk, s0 * np.float32(2.0**k))


def test_negation_flips_sign_bits_only():
    sp = TensorSpec("neg", 200, 300, seed=22, tensor_id=0, sigma=0.02, outlier_p=1e-2)
    x = W.materialize(sp)
    y0, s0 = oracle.quantize(x, sp.M, sp.N)
    y1, s1 = oracle.quantize(x ^ np.uint16(0x8000), sp.M, sp.N)
    assert np.array_equal(y1, y0 ^ np.uint8(0x80))
    assert np.array_equal(s1, s0)


def test_permutation_within_block_permutes_codes():
    rng = np.random.default_rng(9)
    sp = TensorSpec("perm", 128, 256, seed=23, tensor_id=0, sigma=0.02, outlier_p=1e-2)
    x = W.materialize(sp).reshape(128, 256)
    y0, s0 = oracle.quantize(x.ravel(), 128, 256)
    xp = x.copy()
    for bj in range(2):
        blk = x[:, bj * 128:(bj + 1) * 128].ravel()
        p = rng.permutation(blk.size)
        xp[:, bj * 128:(bj + 1) * 128] = blk[p].reshape(128, 128)
        y1, s1 = oracle.quantize(np.ascontiguousarray(xp).ravel(), 128, 256)
        assert np.array_equal(
            y1[:, bj * 128:(bj + 1) * 128].ravel(), y0[:, bj * 128:(bj + 1) * 128].ravel()[p])
        assert np.array_equal(s1, s0)


# ------------------------------------------------------- brute force


def naive_quantize(xf: np.ndarray, bm: int, bn: int):
    """Second quantizer for small shapes: per block, absmax by a full scan,
    scale and reciprocal in binary32, codes by grid search."""
    M, N = xf.shape
    gm, gn = -(-M // bm), -(-N // bn)
    y = np.zeros((M, N), dtype=np.uint8)
    s = np.zeros((gm, gn), dtype=np.float32)
    for bi in range(gm):
        for bj in range(gn):
            blk = xf[bi * bm:(bi + 1) * bm, bj * bn:(bj + 1) * bn]
            a = np.float32(0.0)
            for v in blk.ravel():
                if abs(v) > a:
                    a = np.float32(abs(v))
            a = max(a, EPS)
            sc = np.float32(a) / np.float32(448.0)
            r = np.float32(1.0) / sc
            v = np.clip(blk * r, np.float32(-448), np.float32(448)).astype(np.float32)
            y[bi * bm:(bi + 1) * bm, bj * bn:(bj + 1) * bn] = H.nearest_codes(
                v.astype(np.float64)).reshape(v.shape)
            s[bi, bj] = sc
    return y, s


def test_brute_force_small_workload():
    """The 256x384 small workload (2x3 blocks: all-zero, absmax-448 and x1e-6
    blocks among them) against the naive quantizer, byte for byte."""
    sp = W.small()[0]
    x = W.materialize(sp)
    y, s = oracle.quantize(x, sp.M, sp.N)
    yn, sn = naive_quantize(bf16_bits_to_f32(x).reshape(sp.M, sp.N), 128, 128)
    assert np.array_equal(y, yn)
    assert np.array_equal(s.view(np.uint32), sn.view(np.uint32))
    assert s[1, 0] == 1.0 and (y[0:128, 128:256] == 0).all()


@pytest.mark.parametrize("shape,block", [((130, 129), (128, 128)), ((7, 300), (1, 128)),
                                         ((100, 70), (64, 64)), ((5, 9), (2, 3)),
                                         ((33, 17), (5, 7))])
def test_brute_force_ragged(shape, block):
    M, N = shape
    for dtype in ("bf16", "f32"):
        sp = TensorSpec("rag", M, N, dtype=dtype, seed=31, tensor_id=M * N,
                        dist=DIST_STUDENT_T3, sigma=0.02)
        x = W.materialize(sp)
        y, s = oracle.quantize(x, M, N, bm=block[0], bn=block[1])
        yn, sn = naive_quantize(as_f32(x).reshape(M, N), *block)
        assert np.array_equal(y, yn)
        assert np.array_equal(s.view(np.uint32), sn.view(np.uint32))


def test_row_padding_is_never_read():
    """With ld > N, a large poison value in columns N..ld-1 changes nothing."""
    for dtype in ("bf16", "f32"):
        M, N, ld = 130, 129, 200
        padded = TensorSpec("pad", M, N, ld=ld, dtype=dtype, seed=41, tensor_id=0,
                            dist=DIST_STUDENT_T3, pad_value=3.0e4)
        xp = W.materialize(padded)
        xc = np.ascontiguousarray(xp.reshape(M, ld)[:, :N]).ravel()
        y0, s0 = oracle.quantize(xc, M, N)
        y1, s1 = oracle.quantize(xp, M, N, ld=ld)
        assert np.array_equal(y0, y1) and np.array_equal(s0, s1)
        assert as_f32(xp).reshape(M, ld)[:, N:].min() > 2.9e4


def test_block_api_matches_whole_matrix():
    sp = TensorSpec("blk", 300, 260, seed=51, tensor_id=0, sigma=0.02, outlier_p=1e-2)
    x = W.materialize(sp)
    y, s = oracle.quantize(x, sp.M, sp.N)
    for bi in range(3):
        for bj in range(3):
            yb, sb = oracle.quantize_block(x, sp.M, sp.N, None, 128, 128, bi, bj)
            assert np.array_equal(yb, y[bi * 128:(bi + 1) * 128, bj * 128:(bj + 1) * 128])
            assert sb == s[bi, bj]


def test_rejects_bad_arguments():
    x = np.zeros(16, dtype=np.uint16)
    with pytest.raises(ValueError):
        oracle.quantize(x, 4, 4, ld=3)
    with pytest.raises(ValueError):
        oracle.quantize(x, 4, 8)
    with pytest.raises(TypeError):
        oracle.quantize(np.zeros(16, dtype=np.float64), 4, 4)


def test_golden_order_case_discriminates():
    """The worked example that separates x * (1 / scale) from x / scale: exact
    rational arithmetic confirms that the two orders give different codes, and
    the expected code is the reciprocal-then-multiply one."""
    case = [c for c in json.load(open(GOLDEN))["cases"]
            if c["name"] == "reciprocal_then_multiply_order"][0]
    a, x = (Fraction(float.fromhex(v)) for v in case["x"])
    sc = round_f32(a / 448)
    via_rcp = H.nearest_codes(np.array([float(round_f32(x * round_f32(1 / sc)))]))[0]
    via_div = H.nearest_codes(np.array([float(round_f32(x / sc))]))[0]
    assert via_rcp == int(case["y"][1], 16)
    assert via_div == int(case["y_if_divided_directly"][1], 16)
    assert via_rcp != via_div


# ------------------------------------------------------- dequantization


def test_bf16_rounding_matches_library_cast():
    rng = np.random.default_rng(17)
    pats = rng.integers(0, 2**32, size=1 << 20, dtype=np.uint64).astype(np.uint32)
    v = pats.view(np.float32)
    v = v[np.isfinite(v) & (np.abs(v) < 3.0e38)]
    got = np.array([oracle.lib().fp8bq_oracle_bf16(float(x)) for x in v[:20000]], dtype=np.uint16)
    want = v[:20000].astype(ml_dtypes.bfloat16).view(np.uint16)
    assert np.array_equal(got, want)


def test_dequantize_is_one_rounded_product(random_cases):
    """x_hat = RN_f32(dec(q) * s) exactly; the bf16 output is that value
    rounded to bf16 (nearest even), checked in exact rational arithmetic."""
    from tests.exact import round_bf16
    rng = np.random.default_rng(23)
    for sp, x in random_cases:
        y, s = oracle.quantize(x, sp.M, sp.N)
        xf = oracle.dequantize(y, s, 128, 128, "f32")
        xb = oracle.dequantize(y, s, 128, 128, "bf16")
        d = oracle.e4m3_decode(y)
        for k in rng.integers(0, y.size, size=400):
            r, c = divmod(int(k), sp.N)
            prod = round_f32(frac(d[r, c]) * frac(s[r // 128, c // 128]))
            assert frac(xf[r, c]) == prod
            assert frac(bf16_bits_to_f32(xb[r, c])) == round_bf16(prod)


def test_dequantize_roundtrip_on_grid():
    """Scale 1 (absmax exactly 448): dequantization returns the grid value of
    each code, so every on-grid input comes back exactly."""
    x, q = _grid_block("f32", np.random.default_rng(4))
    y, s = oracle.quantize(x, 128, 128)
    assert s[0, 0] == 1.0
    back = oracle.dequantize(y, s, 128, 128).ravel()
    g = H.grid()
    want = np.where(q & 0x80, -g[q & 0x7F], g[q & 0x7F]).astype(np.float32)
    assert np.array_equal(back, want)
    on = np.isin(np.abs(x).astype(np.float64), g)
    assert on.sum() > 10000 and np.array_equal(back[on], x[on])


def test_dequantize_error_bound(random_cases):
    """|x_hat - x| <= s * ulp_e4m3(x * r) / 2 + one fp32 rounding of each side."""
    for sp, x in random_cases:
        y, s = oracle.quantize(x, sp.M, sp.N)
        xf = as_f32(x).reshape(sp.M, sp.N).astype(np.float64)
        back = oracle.dequantize(y, s, 128, 128).astype(np.float64)
        ss = np.repeat(np.repeat(s.astype(np.float64), 128, 0), 128, 1)[:sp.M, :sp.N]
        r = np.repeat(np.repeat((np.float32(1) / s).astype(np.float64), 128, 0), 128, 1)[:sp.M, :sp.N]
        v = np.clip(xf * r, -448, 448)
        bound = ss * _ulp_e4m3(v.astype(np.float32)) / 2 + (np.abs(xf) + np.abs(back)) * 2.0**-22
        assert (np.abs(back - xf) <= bound).all()


# ------------------------------------------------------- per-tensor scale


def test_tensor_scale_closed_forms():
    """max(max|x|, eps)/448 in exact arithmetic; eps floor on zeros; invariant
    under negation and permutation; equal to the block recipe's descale when
    the tensor is a single block."""
    rng = np.random.default_rng(31)
    for sp in [TensorSpec("t1", 64, 4096, seed=91, tensor_id=1, sigma=1.0, row_lognormal_sigma=1.0),
               TensorSpec("t2", 33, 1000, dtype="f32", seed=91, tensor_id=2, dist=DIST_STUDENT_T3)]:
        x = W.materialize(sp)
        s = oracle.tensor_scale(x)
        a = max(Fraction(float(np.abs(as_f32(x)).max())), frac(EPS))
        assert frac(s) == round_f32(a / 448)
        assert oracle.tensor_scale(x[rng.permutation(x.size)]) == s
        neg = x ^ np.uint16(0x8000) if x.dtype == np.uint16 else -x
        assert oracle.tensor_scale(neg) == s
        y, sb = oracle.quantize(x, 1, x.size, bm=1, bn=x.size)
        assert sb[0, 0] == s
    z = np.zeros(1000, dtype=np.uint16)
    assert frac(oracle.tensor_scale(z)) == round_f32(frac(EPS) / 448)
    assert oracle.tensor_scale(np.array([448.0, -1.0], dtype=np.float32)) == 1.0
