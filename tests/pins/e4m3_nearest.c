/*
 * e4m3_nearest.c -- an independent float8_e4m3fn rounding reference, used only
 * to pin the oracle's bit-manipulation converter.
 *
 * It builds the grid of the 127 non-negative finite e4m3fn values straight
 * from the format (sign 1, exponent 4 with bias 7, mantissa 3, subnormals at
 * exponent field 0, no infinities, S.1111.111 = NaN) in double precision, and
 * rounds by searching that grid: nearest value, and on an exact tie the code
 * whose last bit is 0 (round half to even).  Magnitudes at or above 448
 * saturate to 448.
 *
 * sweep() walks every fp32 bit pattern with a finite magnitude or +-inf,
 * positive and negative, and compares the converter under test with this
 * reference.  Positive patterns increase monotonically in value, so each
 * thread walks its slice with a moving grid index instead of a search.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <string.h>

typedef uint8_t (*conv_fn)(float);

static double grid[127]; /* value of code c, c = 0x00 .. 0x7e */

static void make_grid(void)
{
    for (int c = 0; c < 127; ++c) {
        int efield = c >> 3, m = c & 7;
        grid[c] = efield == 0 ? ldexp((double)m / 8.0, -6)
                              : ldexp(1.0 + (double)m / 8.0, efield - 7);
    }
}

/* nearest grid code for a non-negative double, given i with grid[i] <= a */
static uint8_t round_from(double a, int i)
{
    if (i >= 126)
        return 126;
    double mid = 0.5 * (grid[i] + grid[i + 1]); /* exact in double */
    if (a < mid)
        return (uint8_t)i;
    if (a > mid)
        return (uint8_t)(i + 1);
    return (uint8_t)((i & 1) ? i + 1 : i);
}

typedef struct {
    conv_fn f;
    uint32_t lo, hi; /* positive patterns [lo, hi) */
    uint64_t bad;
    uint32_t first_bad;
    uint8_t first_got, first_want;
} slice;

static void *run_slice(void *arg)
{
    slice *s = (slice *)arg;
    s->bad = 0;
    int i = 0;
    for (uint32_t p = s->lo; p < s->hi; ++p) {
        float v;
        memcpy(&v, &p, 4);
        double a = (double)v;
        while (i < 126 && grid[i + 1] <= a)
            ++i;
        uint8_t want = a >= 448.0 ? 126 : round_from(a, i);
        uint8_t got_p = s->f(v);
        uint8_t got_n = s->f(-v);
        if (got_p != want || got_n != (uint8_t)(want | 0x80)) {
            if (s->bad == 0) {
                s->first_bad = got_p != want ? p : (p | 0x80000000u);
                s->first_got = got_p != want ? got_p : got_n;
                s->first_want = got_p != want ? want : (uint8_t)(want | 0x80);
            }
            s->bad++;
        }
    }
    return NULL;
}

/* Returns the number of mismatching patterns; *first gets the first one as
 * (pattern << 16) | (got << 8) | want. */
uint64_t sweep(conv_fn f, int nthreads, uint64_t *first)
{
    make_grid();
    const uint32_t end = 0x7f800001u; /* +0 .. +inf */
    if (nthreads < 1)
        nthreads = 1;
    if (nthreads > 64)
        nthreads = 64;
    pthread_t th[64];
    slice sl[64];
    for (int t = 0; t < nthreads; ++t) {
        sl[t].f = f;
        sl[t].lo = (uint32_t)((uint64_t)end * t / nthreads);
        sl[t].hi = (uint32_t)((uint64_t)end * (t + 1) / nthreads);
        pthread_create(&th[t], NULL, run_slice, &sl[t]);
    }
    uint64_t bad = 0;
    *first = 0;
    for (int t = 0; t < nthreads; ++t) {
        pthread_join(th[t], NULL);
        if (sl[t].bad && bad == 0)
            *first = ((uint64_t)sl[t].first_bad << 16) | ((uint64_t)sl[t].first_got << 8) |
                     sl[t].first_want;
        bad += sl[t].bad;
    }
    return bad;
}

/* The grid itself, for the tests that need reference values. */
void grid_values(double *out)
{
    make_grid();
    for (int c = 0; c < 127; ++c)
        out[c] = grid[c];
}

/* Reference rounding of an array of doubles (already clamped or not). */
void nearest_codes(const double *v, int64_t n, uint8_t *out)
{
    make_grid();
    for (int64_t k = 0; k < n; ++k) {
        double a = fabs(v[k]);
        uint8_t sign = signbit(v[k]) ? 0x80 : 0;
        uint8_t code;
        if (a >= 448.0) {
            code = 126;
        } else {
            int lo = 0, hi = 126; /* grid[lo] <= a < grid[hi] */
            while (hi - lo > 1) {
                int mid = (lo + hi) / 2;
                if (grid[mid] <= a)
                    lo = mid;
                else
                    hi = mid;
            }
            code = round_from(a, lo);
        }
        out[k] = (uint8_t)(sign | code);
    }
}
