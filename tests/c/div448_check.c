/*
 * The kernels compute a block's scale s = a / 448 without a division:
 *     z = RN(1/448),  q0 = RN(a * z),  s = RN(q0 + RN(a - 448 * q0) * z)
 * (the two last steps as fused multiply-adds; Brisebarre, Muller and Raina,
 * "Accelerating correctly rounded floating-point division when the divisor is
 * known in advance", IEEE Trans. Computers 53(8), 2004).  That method is
 * correctly rounded for every dividend only for some divisors, so this
 * program checks it against IEEE division for every float a from the eps
 * floor (1e-10f, the smallest absmax a block can have) to FLT_MAX.
 * Prints the count and exits 1 on the first difference.
 */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>

static float from_bits(uint32_t u) {
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

static uint32_t to_bits(float f) {
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    return u;
}

int main(void) {
    const float b = 448.0f;
    const volatile float one = 1.0f;  /* keep 1/448 an IEEE run-time division */
    const float z = one / b;
    const uint32_t lo = to_bits(1e-10f), hi = to_bits(3.40282347e38f);
    uint64_t n = 0;
    for (uint32_t bits = lo;; ++bits) {
        const float a = from_bits(bits);
        const float q0 = a * z;
        const float s = fmaf(fmaf(-q0, b, a), z, q0);
        const float want = a / b;
        ++n;
        if (to_bits(s) != to_bits(want)) {
            printf("a = %a: %a, IEEE division %a\n", a, s, want);
            return 1;
        }
        if (bits == hi) break;
    }
    printf("%llu dividends, all correctly rounded\n", (unsigned long long)n);
    return 0;
}
