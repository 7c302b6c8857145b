/*
 * Exhaustive check of the oracle's fp32 -> E4M3 and fp32 -> E2M1 nearest-even
 * rounding over all 2^32 fp32 bit patterns (test infrastructure).
 *
 * The reference here is written independently of the oracle: the non-negative
 * finite grid of each format is listed from its bit layout (E4M3: bias 7,
 * 3 mantissa bits, largest 448 = 0x7E; E2M1: bias 1, 1 mantissa bit, largest
 * 6 = 0x7), the nearest grid value is found by binary search on |v| in
 * double, a tie goes to the even code, magnitudes beyond the largest value
 * saturate to it, NaN gives 0x7F (E4M3) / 0x7 (E2M1), and the sign bit is
 * copied from v.  Prints "mismatches <e4m3> <e2m1>" and returns 0 when both
 * are zero.
 */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>

uint8_t oracle_e4m3_rne(float v);
uint8_t oracle_e2m1_rne(float v);

static double g8[127], g4[8];

static void grids(void) {
    for (int c = 0; c < 127; ++c) {
        int e = c >> 3, m = c & 7;
        g8[c] = e == 0 ? ldexp((double)m, -9) : ldexp(1.0 + m / 8.0, e - 7);
    }
    for (int c = 0; c < 8; ++c) {
        int e = c >> 1, m = c & 1;
        g4[c] = e == 0 ? 0.5 * m : ldexp(1.0 + m / 2.0, e - 1);
    }
}

static int nearest(const double *g, int n, double a) {
    if (a >= g[n - 1]) return n - 1;
    int lo = 0, hi = n - 1;                 /* g[lo] <= a < g[hi] */
    while (hi - lo > 1) {
        int mid = (lo + hi) / 2;
        if (g[mid] <= a) lo = mid; else hi = mid;
    }
    double dl = a - g[lo], dh = g[hi] - a;
    if (dl < dh) return lo;
    if (dh < dl) return hi;
    return (lo & 1) ? hi : lo;              /* tie: the even code */
}

int main(void) {
    grids();
    unsigned long long bad8 = 0, bad4 = 0;
#pragma omp parallel for reduction(+ : bad8, bad4) schedule(static)
    for (long long i = 0; i < (1LL << 32); ++i) {
        uint32_t b = (uint32_t)i;
        float v;
        memcpy(&v, &b, 4);
        uint8_t s8 = (b >> 31) ? 0x80 : 0, s4 = (b >> 31) ? 0x8 : 0;
        uint8_t r8, r4;
        if (isnan(v)) {
            r8 = s8 | 0x7F;
            r4 = s4 | 0x7;
        } else {
            double a = fabs((double)v);
            r8 = s8 | (uint8_t)nearest(g8, 127, a);
            r4 = s4 | (uint8_t)nearest(g4, 8, a);
        }
        if (oracle_e4m3_rne(v) != r8) ++bad8;
        if (oracle_e2m1_rne(v) != r4) ++bad4;
    }
    printf("mismatches %llu %llu\n", bad8, bad4);
    return (bad8 || bad4) ? 1 : 0;
}
