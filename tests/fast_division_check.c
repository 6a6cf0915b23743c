/*
 * Exhaustive check of the quotient the group-quantisation kernel forms in
 * place of an IEEE fp32 divide by an E4M3 scale (and by 3 for the scale
 * itself): with y = RN(1/M), q0 = RN(a*y), r = fma(-M, q0, a) (exact) and
 * q = fma(r, y, q0), Markstein's correction step, the result is compared
 * with the IEEE quotient RN(a/M) for every finite fp32 a and every E4M3
 * significand M in 1..15 (an E4M3 value is M * 2^e; scaling by 2^e is exact
 * for the quotients that matter, |a/s| < 2^120, away from subnormals).
 *
 * Exit 0 and print "ok" when q == RN(a/M) for every a whose quotient is a
 * normal float, and both are below 2^-10 in magnitude otherwise (there the
 * E4M3 rounding and the 2-bit code are 0 for either).
 *
 * Modes: "all" walks every fp32 bit pattern (about 5 minutes on 8 cores);
 * the default walks every a with a/M in [1, 2) and both signs.  Multiplying
 * a by 2^k scales q0, r and q by 2^k exactly while every value stays normal,
 * so one binade of quotients stands for every normal quotient.
 *
 * Build: gcc -O2 -ffp-contract=off -fopenmp fast_division_check.c -lm
 */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>

static float bits_to_f(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }
static uint32_t f_to_bits(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }

int main(int argc, char** argv) {
    const int all = argc > 1 && strcmp(argv[1], "all") == 0;
    long long bad = 0, checked = 0, tiny = 0;
    for (int M = 1; M <= 15; ++M) {
        const float fm = (float)M;
        const float y = 1.0f / fm;                      /* RN(1/M) */
        /* default range: bit patterns of [M, 2M) (a/M in [1, 2)), both signs */
        const long long lo = all ? 0 : (long long)f_to_bits(fm);
        const long long hi = all ? (1LL << 32) : (long long)f_to_bits(2.0f * fm);
        long long bad_m = 0, checked_m = 0, tiny_m = 0;
#pragma omp parallel for reduction(+ : bad_m, checked_m, tiny_m) schedule(static)
        for (long long j = 0; j < (all ? hi : 2 * (hi - lo)); ++j) {
            const uint32_t i = all ? (uint32_t)j : (uint32_t)(lo + j / 2) | (j & 1 ? 0x80000000u : 0u);
            const float a = bits_to_f(i);
            if (!isfinite(a)) continue;
            const float exact = a / fm;
            const float q0 = a * y;
            const float r = fmaf(-fm, q0, a);
            const float q = fmaf(r, y, q0);
            ++checked_m;
            if (fabsf(exact) >= 0x1p-126f) {
                if (f_to_bits(q) != f_to_bits(exact)) ++bad_m;
            } else {
                ++tiny_m;
                if (!(fabsf(q) < 0x1p-10f)) ++bad_m;
            }
        }
        if (bad_m) printf("M=%d: %lld mismatches\n", M, bad_m);
        bad += bad_m; checked += checked_m; tiny += tiny_m;
    }
    printf("%s checked=%lld subnormal_quotients=%lld mismatches=%lld\n", bad ? "FAIL" : "ok", checked, tiny, bad);
    return bad ? 1 : 0;
}
