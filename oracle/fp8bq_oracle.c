/*
 * fp8bq_oracle.c -- CPU oracle for the blockwise FP8 (float8_e4m3fn) weight
 * quantizer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path links, loads or
 * calls this file: only the tests, the smoke check and the benchmark's
 * cpu_baseline / reference legs do.  It shares no code, header, table or
 * constant generator with the CUDA library; the two meet only through the
 * seeded inputs of the synthetic-workload generator.
 *
 * It is deliberately plain: single-threaded, one block at a time, one element
 * at a time, in the order the method states its steps.  Floating point is IEEE
 * binary32 with round-to-nearest-even, because that is the precision the
 * method itself computes in (the kernel's absmax, scale, reciprocal and
 * product are fp32 values and the descale it stores is fp32).  Build with
 * -ffp-contract=off and without fast-math so that the compiler neither fuses
 * the multiply nor flushes subnormals.
 *
 * Sources (verl documentation and review pages on FP8 rollout):
 *   [K1] "fp8_kernel.py -- FP8 量化内核" (verl/utils/kernel/fp8_kernel.py docs),
 *        section 1 "统一入口" (scaled_fp8_blockwise: [M,N] input,
 *        [BLOCK_M, BLOCK_N] block size, returns (fp8_data, descale)).
 *   [K2] same page, section 2 "Triton 实现": per block, absmax of |x| floored
 *        by eps; x_s = absmax / fp8_max; y = clamp(x * (1 / x_s), fp8_min,
 *        fp8_max); store y into the fp8 tensor and x_s into the scale tensor.
 *   [K3] same page, section 3 "PyTorch Fallback": per-block abs().amax, then
 *        multiply, clamp to +-max and cast .to(float8_e4m3fn).
 *   [K4] same page, "背景知识": the format is float8_e4m3fn.
 *   [U3] "vllm_fp8_utils.py" docs, section 3 "权重量化": the descale is emitted
 *        as "<name>_scale_inv" next to the fp8 weight.
 *   [P1] "FP8-RL: A Practical and Stable Low-Precision Stack for LLM
 *        Reinforcement Learning", abstract: the KV cache is also FP8, with its
 *        Q/K/V scales recalibrated every RL step.
 *
 * Readings taken where the pages are silent (each is listed in the design
 * notes):
 *   - eps is a parameter of every entry point here; the library fixes it at
 *     1e-10f.
 *   - fp8_min / fp8_max are -448 / +448, the finite range of float8_e4m3fn.
 *   - both divisions are IEEE round-to-nearest; the order is div, div, mul.
 *   - the store's fp32 -> e4m3fn conversion rounds to nearest, ties to even,
 *     and saturates to +-448; the sign of a result that rounds to zero is kept.
 *   - an edge block takes its absmax over its valid elements only and writes
 *     only its valid elements.
 *   - the fp8 output is a contiguous row-major [M, N]; the descale is a
 *     contiguous row-major [ceil(M/BLOCK_M), ceil(N/BLOCK_N)] fp32 array.
 *
 * Parity pins (tests under -m "not gpu") check every function here against
 * facts the pages and the format fix: an exhaustive sweep of the converter
 * over all finite fp32 bit patterns against a nearest-value search of the
 * e4m3fn grid, directed blocks (all zero, absmax exactly 448, the whole e4m3
 * grid), exact-rational checks of the scale, metamorphic invariants and a
 * brute-force second quantizer on small shapes.
 */
#include <stdint.h>
#include <stddef.h>
#include <string.h>

#define ORACLE_DTYPE_BF16 0
#define ORACLE_DTYPE_F32 1

/* Largest finite float8_e4m3fn magnitude: exponent field 1111, mantissa 110,
 * i.e. 1.75 * 2^(15-7) = 448 ([K4], read from the e4m3fn format). */
static const float E4M3_MAX = 448.0f;

static float f32_from_bits(uint32_t b)
{
    float f;
    memcpy(&f, &b, sizeof f);
    return f;
}

static uint32_t bits_from_f32(float f)
{
    uint32_t b;
    memcpy(&b, &f, sizeof b);
    return b;
}

/* Element (r, c) of a row-major matrix with row stride ld (in elements),
 * widened to fp32.  bf16 is the upper half of an fp32, so widening is exact. */
static float load_elem(const void *x, int dtype, int64_t ld, int64_t r, int64_t c)
{
    int64_t i = r * ld + c;
    if (dtype == ORACLE_DTYPE_BF16) {
        uint16_t h = ((const uint16_t *)x)[i];
        return f32_from_bits((uint32_t)h << 16);
    }
    return ((const float *)x)[i];
}

/*
 * fp32 -> float8_e4m3fn, round to nearest with ties to even, saturating to
 * +-448 ([K2] store of y into the fp8 tensor; [K3] .to(float8_e4m3fn) after the
 * clamp; [K4] format).  e4m3fn: 1 sign bit, 4 exponent bits with bias 7,
 * 3 mantissa bits, no infinities, S.1111.111 is NaN.  Normal values are
 * (1 + m/8) * 2^(E-7) for E in 1..15 (E=15, m=7 excluded); subnormals are
 * (m/8) * 2^-6 = m * 2^-9.
 */
uint8_t fp8bq_oracle_e4m3(float v)
{
    uint32_t b = bits_from_f32(v);
    uint8_t sign = (uint8_t)((b >> 31) << 7);
    uint32_t mag = b & 0x7fffffffu;

    if (mag > 0x7f800000u) /* NaN in, NaN out; outside the method's contract */
        return (uint8_t)(sign | 0x7f);

    float a = f32_from_bits(mag);
    if (a >= E4M3_MAX) /* saturate, +-inf included */
        return (uint8_t)(sign | 0x7e);

    if (a >= 0.015625f) { /* normal range, a >= 2^-6 */
        int e = (int)(mag >> 23) - 127;    /* unbiased exponent, -6..8 */
        uint32_t m = mag & 0x7fffffu;      /* 23 fp32 mantissa bits */
        uint32_t q = m >> 20;              /* top 3 kept */
        uint32_t rest = m & 0xfffffu;      /* 20 dropped */
        uint32_t code = ((uint32_t)(e + 7) << 3) | q;
        if (rest > 0x80000u || (rest == 0x80000u && (q & 1u)))
            code += 1; /* a mantissa carry moves into the exponent field */
        if (code > 0x7eu) /* would be 480 or NaN: saturate */
            code = 0x7eu;
        return (uint8_t)(sign | code);
    }

    /* Subnormal range: the grid is k * 2^-9, k = 0..8 (k = 8 is 2^-6, the
     * smallest normal, whose code is also 8).  a * 512 is exact. */
    float t = a * 512.0f;
    uint32_t k = (uint32_t)t;        /* floor, t in [0, 8) */
    float frac = t - (float)k;       /* exact */
    if (frac > 0.5f || (frac == 0.5f && (k & 1u)))
        k += 1;
    return (uint8_t)(sign | k);
}

/* float8_e4m3fn -> fp32 (exact).  Used for dequantization x_hat = dec(q) * s,
 * the meaning of the "_scale_inv" tensor ([U3]). */
float fp8bq_oracle_e4m3_decode(uint8_t q)
{
    uint32_t sign = (uint32_t)(q >> 7);
    uint32_t e = (uint32_t)((q >> 3) & 0xf);
    uint32_t m = (uint32_t)(q & 7);
    float mag;
    if (e == 15 && m == 7) {
        mag = f32_from_bits(0x7fc00000u); /* NaN */
    } else if (e == 0) {
        mag = (float)m * 0.001953125f; /* m * 2^-9, exact */
    } else {
        /* (8 + m) * 2^(e - 10), exact */
        float p = 1.0f;
        int k = (int)e - 10;
        for (; k > 0; --k) p *= 2.0f;
        for (; k < 0; ++k) p *= 0.5f;
        mag = (float)(8 + m) * p;
    }
    return sign ? -mag : mag;
}

/*
 * One block (bi, bj) of an [M, N] matrix ([K2]: one Triton program per block,
 * program ids (pid_m, pid_n)).  The block covers rows bi*bm .. and columns
 * bj*bn .., clipped to the matrix.  Writes the block's fp8 codes to
 * y_blk[r * ldy + c] for the block-local valid (r, c), and its descale to
 * *s_out.
 */
void fp8bq_oracle_block(const void *x, int dtype, int64_t M, int64_t N, int64_t ld,
                        int bm, int bn, float eps, int64_t bi, int64_t bj,
                        uint8_t *y_blk, int64_t ldy, float *s_out)
{
    int64_t r0 = bi * (int64_t)bm, c0 = bj * (int64_t)bn;
    int64_t rows = M - r0 < bm ? M - r0 : bm;
    int64_t cols = N - c0 < bn ? N - c0 : bn;

    /* step 1: absmax over the valid elements, then the eps floor ([K2]) */
    float amax = 0.0f;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t c = 0; c < cols; ++c) {
            float ax = load_elem(x, dtype, ld, r0 + r, c0 + c);
            ax = ax < 0.0f ? -ax : ax;
            if (ax > amax)
                amax = ax;
        }
    if (amax < eps)
        amax = eps;

    /* step 2: scale = absmax / fp8_max, step 3: its reciprocal ([K2]) */
    float s = amax / E4M3_MAX;
    float rcp = 1.0f / s;

    /* step 4: multiply, clamp to [-448, 448], convert ([K2], [K3]) */
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t c = 0; c < cols; ++c) {
            float v = load_elem(x, dtype, ld, r0 + r, c0 + c) * rcp;
            if (v > E4M3_MAX)
                v = E4M3_MAX;
            else if (v < -E4M3_MAX)
                v = -E4M3_MAX;
            y_blk[r * ldy + c] = fp8bq_oracle_e4m3(v);
        }

    /* step 5: the stored descale is the scale itself ([K2] stores x_s) */
    *s_out = s;
}

/*
 * Whole matrix ([K1]: scaled_fp8_blockwise(data_hp, weight_block_size)).
 * x: [M, N] with row stride ld >= N elements; y: contiguous [M, N] bytes;
 * s: contiguous [ceil(M/bm), ceil(N/bn)] floats.  Returns 0, or -1 on an
 * argument it cannot handle.
 */
int fp8bq_oracle_quantize(const void *x, int dtype, int64_t M, int64_t N, int64_t ld,
                          int bm, int bn, float eps, uint8_t *y, float *s)
{
    if (M < 0 || N < 0 || ld < N || bm < 1 || bn < 1)
        return -1;
    if (dtype != ORACLE_DTYPE_BF16 && dtype != ORACLE_DTYPE_F32)
        return -1;
    int64_t gm = (M + bm - 1) / bm, gn = (N + bn - 1) / bn;
    for (int64_t bi = 0; bi < gm; ++bi)
        for (int64_t bj = 0; bj < gn; ++bj)
            fp8bq_oracle_block(x, dtype, M, N, ld, bm, bn, eps, bi, bj,
                               y + bi * bm * N + bj * bn, N, s + bi * gn + bj);
    return 0;
}

/* Element-wise converter and decoder over arrays, for the pins. */
void fp8bq_oracle_e4m3_array(const float *v, int64_t n, uint8_t *out)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = fp8bq_oracle_e4m3(v[i]);
}

void fp8bq_oracle_e4m3_decode_array(const uint8_t *q, int64_t n, float *out)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = fp8bq_oracle_e4m3_decode(q[i]);
}

/*
 * Dequantization, the consumer side of the "_scale_inv" tensor ([U3]): the
 * descale is the multiplier that maps codes back to weights,
 *     x_hat[r, c] = dec(y[r, c]) * s[r / bm, c / bn]
 * with one fp32 multiply (round to nearest even).  The pages print no
 * dequantization code; this is the plain reading of the descale's meaning.
 */
void fp8bq_oracle_dequantize(const uint8_t *y, const float *s, int64_t M, int64_t N,
                             int bm, int bn, float *out)
{
    int64_t gn = (N + bn - 1) / bn;
    for (int64_t r = 0; r < M; ++r)
        for (int64_t c = 0; c < N; ++c)
            out[r * N + c] = fp8bq_oracle_e4m3_decode(y[r * N + c]) * s[(r / bm) * gn + c / bn];
}

/* fp32 -> bf16 bits, round to nearest, ties to even (finite inputs). */
uint16_t fp8bq_oracle_bf16(float v)
{
    uint32_t b = bits_from_f32(v);
    uint32_t keep = b >> 16, rest = b & 0xffffu;
    if (rest > 0x8000u || (rest == 0x8000u && (keep & 1u)))
        keep += 1; /* a carry into the exponent is the correct rounding */
    return (uint16_t)keep;
}

/* Dequantization to bf16: the fp32 product above, rounded to bf16. */
void fp8bq_oracle_dequantize_bf16(const uint8_t *y, const float *s, int64_t M, int64_t N,
                                  int bm, int bn, uint16_t *out)
{
    int64_t gn = (N + bn - 1) / bn;
    for (int64_t r = 0; r < M; ++r)
        for (int64_t c = 0; c < N; ++c)
            out[r * N + c] = fp8bq_oracle_bf16(fp8bq_oracle_e4m3_decode(y[r * N + c]) *
                                               s[(r / bm) * gn + c / bn]);
}

/*
 * Per-tensor scale of the FP8 KV cache, recalibrated each step ([P1]): the
 * pages name the recalibration but print no formula; the reading is the
 * weight recipe ([K2]) applied to the whole tensor as one block,
 *     s = max(max |x|, eps) / 448
 * (fp32, round to nearest).  x holds numel contiguous elements.
 */
float fp8bq_oracle_tensor_scale(const void *x, int dtype, int64_t numel, float eps)
{
    float amax = 0.0f;
    for (int64_t i = 0; i < numel; ++i) {
        float ax = load_elem(x, dtype, 0, 0, i);
        ax = ax < 0.0f ? -ax : ax;
        if (ax > amax)
            amax = ax;
    }
    if (amax < eps)
        amax = eps;
    return amax / E4M3_MAX;
}
