/*
 * synth.c -- seeded synthetic weight matrices for tests and benchmarks.
 *
 * This file holds input preparation only: random numbers, value
 * distributions, and the rounding of the composed values to the storage type.
 * It contains none of the quantizer's arithmetic.  Both the CPU oracle and the
 * CUDA library read the buffers it writes, so the two always see identical
 * inputs.
 *
 * Generator: SplitMix64 (Steele, Lea and Flood, "Fast Splittable Pseudorandom
 * Number Generators", OOPSLA 2014) used in counter mode: the n-th output of a
 * stream with key k is mix(k + n * 0x9E3779B97F4A7C15), where mix is the
 * SplitMix64 output function.  Every element's random numbers are a pure
 * function of (seed, tensor id, stream tag, element index), so the result
 * does not depend on thread count or fill order.
 *
 * Normals: Box-Muller in double, with the two outputs of one pair of uniforms
 * serving two neighbouring elements.  Values are composed in double, rounded
 * to fp32 (round to nearest), and for bf16 storage rounded again to bf16
 * (round to nearest, ties to even).
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <string.h>

#define GOLDEN_GAMMA 0x9E3779B97F4A7C15ull

static inline uint64_t sm64_mix(uint64_t z)
{
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

/* n-th output of the SplitMix64 stream whose state starts at key */
static inline uint64_t sm64_at(uint64_t key, uint64_t n)
{
    return sm64_mix(key + (n + 1) * GOLDEN_GAMMA);
}

/* Stream key for (seed, tensor id, tag). */
static uint64_t stream_key(uint64_t seed, uint64_t tensor, uint64_t tag)
{
    uint64_t k = sm64_at(seed, 0);
    k = sm64_at(k ^ tensor, 1);
    return sm64_at(k ^ (tag << 32), 2);
}

/* uniform in the open interval (0, 1) from the top 53 bits */
static inline double u01(uint64_t r)
{
    return ((double)(r >> 11) + 0.5) * (1.0 / 9007199254740992.0);
}

/* standard normal for counter n of the stream, Box-Muller over pairs */
static inline double normal_at(uint64_t key, uint64_t n)
{
    uint64_t p = n >> 1;
    double u1 = u01(sm64_at(key, 2 * p));
    double u2 = u01(sm64_at(key, 2 * p + 1));
    double rad = sqrt(-2.0 * log(u1));
    double th = 6.283185307179586 * u2;
    return (n & 1) ? rad * sin(th) : rad * cos(th);
}

static inline uint16_t bf16_rne(float f)
{
    uint32_t b;
    memcpy(&b, &f, 4);
    if ((b & 0x7f800000u) == 0x7f800000u) /* inf / nan: truncate, keep nan quiet */
        return (uint16_t)((b >> 16) | ((b & 0xffffu) ? 0x40u : 0u));
    b += 0x7fffu + ((b >> 16) & 1u);
    return (uint16_t)(b >> 16);
}

enum { DIST_NORMAL = 0, DIST_STUDENT_T3 = 1 };
enum { TAG_VALUE = 1, TAG_ROW = 2, TAG_BATCH = 3, TAG_OUTLIER = 4, TAG_CHI = 5 };

typedef struct {
    uint64_t seed;
    uint64_t tensor_id;
    int64_t batch, M, N, ld, batch_stride; /* in elements; ld >= N */
    int32_t dtype;                         /* 0: bf16 bits, 1: fp32 */
    int32_t dist;                          /* DIST_* */
    double sigma;                          /* overall scale */
    double row_lognormal_sigma;            /* per (batch, row) factor exp(s*z); 0 = off */
    double batch_lognormal_sigma;          /* per batch factor exp(s*z); 0 = off */
    double outlier_p, outlier_lo, outlier_hi; /* |x| ~ U(lo, hi) with prob p */
    double pad_value;                      /* written to columns N..ld-1 */
    int32_t nthreads;
} synth_spec;

typedef struct {
    const synth_spec *sp;
    void *out;
    int64_t el_begin, el_end; /* over the batch*M*N logical elements, row-major */
} job;

static double value_at(const synth_spec *sp, uint64_t kv, uint64_t kc, uint64_t ko,
                       double factor, uint64_t e)
{
    double v;
    if (sp->dist == DIST_STUDENT_T3) {
        double z0 = normal_at(kv, e);
        double z1 = normal_at(kc, 3 * e), z2 = normal_at(kc, 3 * e + 1),
               z3 = normal_at(kc, 3 * e + 2);
        v = z0 / sqrt((z1 * z1 + z2 * z2 + z3 * z3) / 3.0);
    } else {
        v = normal_at(kv, e);
    }
    v *= sp->sigma * factor;
    if (sp->outlier_p > 0.0) {
        uint64_t r = sm64_at(ko, 2 * e);
        if (u01(r) < sp->outlier_p) {
            double m = sp->outlier_lo + (sp->outlier_hi - sp->outlier_lo) * u01(sm64_at(ko, 2 * e + 1));
            v = (r & 1) ? -m : m;
        }
    }
    return v;
}

static void *run_job(void *arg)
{
    const job *jb = (const job *)arg;
    const synth_spec *sp = jb->sp;
    uint64_t kv = stream_key(sp->seed, sp->tensor_id, TAG_VALUE);
    uint64_t kr = stream_key(sp->seed, sp->tensor_id, TAG_ROW);
    uint64_t kb = stream_key(sp->seed, sp->tensor_id, TAG_BATCH);
    uint64_t ko = stream_key(sp->seed, sp->tensor_id, TAG_OUTLIER);
    uint64_t kc = stream_key(sp->seed, sp->tensor_id, TAG_CHI);
    float pad = (float)sp->pad_value;
    /* the rows this job's element range touches; a row's padding columns are
     * written by the job that holds the row's last element */
    for (int64_t fr = jb->el_begin / sp->N; fr * sp->N < jb->el_end; ++fr) {
        int64_t b = fr / sp->M, r = fr % sp->M;
        double factor = 1.0;
        if (sp->batch_lognormal_sigma != 0.0)
            factor *= exp(sp->batch_lognormal_sigma * normal_at(kb, (uint64_t)b));
        if (sp->row_lognormal_sigma != 0.0)
            factor *= exp(sp->row_lognormal_sigma * normal_at(kr, (uint64_t)fr));
        int64_t base = b * sp->batch_stride + r * sp->ld;
        uint64_t e0 = (uint64_t)fr * (uint64_t)sp->N; /* logical element index */
        int64_t c0 = jb->el_begin > fr * sp->N ? jb->el_begin - fr * sp->N : 0;
        int64_t c1 = jb->el_end < (fr + 1) * sp->N ? jb->el_end - fr * sp->N : sp->N;
        int64_t p1 = c1 == sp->N ? sp->ld : c1;
        if (sp->dtype == 0) {
            uint16_t *o = (uint16_t *)jb->out + base;
            for (int64_t c = c0; c < c1; ++c)
                o[c] = bf16_rne((float)value_at(sp, kv, kc, ko, factor, e0 + (uint64_t)c));
            for (int64_t c = c1; c < p1; ++c)
                o[c] = bf16_rne(pad);
        } else {
            float *o = (float *)jb->out + base;
            for (int64_t c = c0; c < c1; ++c)
                o[c] = (float)value_at(sp, kv, kc, ko, factor, e0 + (uint64_t)c);
            for (int64_t c = c1; c < p1; ++c)
                o[c] = pad;
        }
    }
    return NULL;
}

/* Fill out[b * batch_stride + r * ld + c] for all b, r < M, c < ld.
 * Returns 0 on success, -1 on bad arguments. */
int synth_fill(const synth_spec *sp, void *out)
{
    if (sp->batch < 0 || sp->M < 0 || sp->N < 0 || sp->ld < sp->N)
        return -1;
    int64_t rows = sp->batch * sp->M;
    if (rows == 0 || sp->ld == 0)
        return 0;
    if (sp->N == 0) { /* rows of padding only */
        for (int64_t fr = 0; fr < rows; ++fr) {
            int64_t base = (fr / sp->M) * sp->batch_stride + (fr % sp->M) * sp->ld;
            for (int64_t c = 0; c < sp->ld; ++c) {
                if (sp->dtype == 0)
                    ((uint16_t *)out)[base + c] = bf16_rne((float)sp->pad_value);
                else
                    ((float *)out)[base + c] = (float)sp->pad_value;
            }
        }
        return 0;
    }
    /* threads split the logical elements evenly (values depend only on the
     * element's index, so any split gives the same array): long rows of
     * few-row tensors are shared too */
    int64_t total = rows * sp->N;
    int nt = sp->nthreads < 1 ? 1 : sp->nthreads;
    if (nt > 256)
        nt = 256;
    if (total < (int64_t)nt * 4096)
        nt = (int)(total / 4096) > 0 ? (int)(total / 4096) : 1;
    pthread_t th[256];
    job jobs[256];
    for (int t = 0; t < nt; ++t) {
        jobs[t].sp = sp;
        jobs[t].out = out;
        jobs[t].el_begin = (int64_t)((__int128)total * t / nt);
        jobs[t].el_end = (int64_t)((__int128)total * (t + 1) / nt);
    }
    int started = 0;
    for (int t = 1; t < nt; ++t) {
        if (pthread_create(&th[t], NULL, run_job, &jobs[t]) != 0)
            break;
        started = t;
    }
    run_job(&jobs[0]);
    for (int t = 1; t <= started; ++t)
        pthread_join(th[t], NULL);
    for (int t = started + 1; t < nt; ++t) /* threads that could not start */
        run_job(&jobs[t]);
    return 0;
}

/* fp32 -> bf16 bit patterns, round to nearest even (input preparation). */
void synth_f32_to_bf16(const float *in, int64_t n, uint16_t *out)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = bf16_rne(in[i]);
}
