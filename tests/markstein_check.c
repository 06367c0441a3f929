/* Markstein's division from a correctly rounded reciprocal, against IEEE
 * float division: for b with y = RN(1/b),
 *     q0 = RN(x * y);  e = RN(x - b * q0) (one FMA, exact);  q1 = RN(q0 + e * y)
 * must equal RN(x / b) whenever the remainder x - b * q0 is representable.
 * Checks every dividend mantissa x in [1, 2) against nb divisors in [1, 2)
 * and [2, 4) (edge significands first, then a xorshift sequence); scaling
 * by powers of two carries the result to every exponent at which the
 * remainder stays representable, i.e. quotients well above 2^-126 * 2^24.
 * Nearer underflow the remainder can need bits below 2^-149 (and a
 * subnormal dividend never has an exact one: the second mode shows it).  Prints the
 * count of quotients and of mismatches.  Build: gcc -O2 -std=c11
 * -ffp-contract=off -fno-fast-math -fopenmp markstein_check.c -lm */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

static float fbits(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }
static uint32_t bits(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }

int main(int argc, char **argv) {
    const int nb = argc > 1 ? atoi(argv[1]) : 64;
    const int subnormal = argc > 2 ? atoi(argv[2]) : 0;  /* 1: subnormal dividends instead */
    static const uint32_t edges[] = {0x3f800000u, 0x3f800001u, 0x3fffffffu, 0x3fc00000u,
                                     0x3fbfffffu, 0x3fb504f3u, 0x3f800002u, 0x3ffffffeu};
    uint32_t *bs = malloc(sizeof(uint32_t) * (size_t)(nb + 8));
    int n = 0;
    for (int i = 0; i < 8 && n < nb; ++i) bs[n++] = edges[i];
    uint64_t st = 88172645463325252ull;
    while (n < nb) {
        st ^= st << 13; st ^= st >> 7; st ^= st << 17;
        bs[n++] = 0x3f800000u | (uint32_t)(st & 0x7fffffu);
    }
    unsigned long long total = 0, bad = 0;
#pragma omp parallel for reduction(+ : total, bad) schedule(dynamic)
    for (int ib = 0; ib < n; ++ib)
        for (int eb = 0; eb < 2; ++eb) {
            /* normal dividends: b in [1, 2) or [2, 4); subnormal ones: b in [1/2, 1) or [1/4, 1/2) */
            const float b = subnormal ? fbits(bs[ib] - ((uint32_t)(eb + 1) << 23)) : fbits(bs[ib] + ((uint32_t)eb << 23));
            const float y = 1.0f / b;
            for (uint32_t m = subnormal ? 1u : 0u; m < (1u << 23); ++m) {
                const float x = subnormal ? fbits(m) : fbits(0x3f800000u | m);
                const float q0 = x * y;
                const float q1 = fmaf(fmaf(-q0, b, x), y, q0);
                total++;
                if (bits(q1) != bits(x / b)) bad++;
            }
        }
    printf("%llu %llu\n", total, bad);
    free(bs);
    return 0;
}
