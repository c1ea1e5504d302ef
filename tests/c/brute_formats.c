/*
 * Exhaustive check of the oracle's E2M1 and E4M3 rounding against a separate
 * brute-force search, over every fp32 bit pattern (NaNs skipped).
 *
 * The brute force knows only the format definitions: it lists the finite
 * values of each format, takes the nearest one to |x| (exact in double), and
 * breaks a tie towards the code whose last mantissa bit is 0.  A magnitude at
 * or beyond the largest finite value maps to that value (it is the nearest).
 *
 * usage: brute_formats <path to oracle .so>   (prints mismatch counts)
 */
#include <dlfcn.h>
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>

typedef uint32_t (*enc_fn)(float);

static double e2m1_grid[8];
static double e4m3_grid[127];

static uint32_t brute_e2m1(float x)
{
    double a = fabs((double)x);
    /* at or beyond the largest value the nearest point is the largest value;
       handled first because a - 4 and a - 6 are equal in double for huge a */
    if (a >= e2m1_grid[7]) return (signbit(x) ? 8u : 0u) | 7u;
    int best = 0;
    double bd = fabs(a - e2m1_grid[0]);
    for (int i = 1; i < 8; ++i) {
        double d = fabs(a - e2m1_grid[i]);
        if (d < bd || (d == bd && (i & 1) == 0 && (best & 1) == 1)) { bd = d; best = i; }
    }
    return (signbit(x) ? 8u : 0u) | (uint32_t)best;
}

static uint32_t brute_e4m3(float x)
{
    double a = fabs((double)x);
    /* largest grid index with value <= a (grid ascending) */
    int lo = 0, hi = 126;
    if (a >= e4m3_grid[126]) return (signbit(x) ? 0x80u : 0u) | 126u;
    while (hi - lo > 1) {
        int mid = (lo + hi) / 2;
        if (e4m3_grid[mid] <= a) lo = mid; else hi = mid;
    }
    double dl = a - e4m3_grid[lo], dh = e4m3_grid[hi] - a;
    int best = (dl < dh) ? lo : (dh < dl) ? hi : ((lo & 1) == 0 ? lo : hi);
    return (signbit(x) ? 0x80u : 0u) | (uint32_t)best;
}

int main(int argc, char** argv)
{
    if (argc < 2) return 2;
    void* h = dlopen(argv[1], RTLD_NOW);
    if (!h) { fprintf(stderr, "%s\n", dlerror()); return 2; }
    enc_fn o_e2m1 = (enc_fn)dlsym(h, "oracle_e2m1_encode");
    enc_fn o_e4m3 = (enc_fn)dlsym(h, "oracle_e4m3_encode");
    if (!o_e2m1 || !o_e4m3) return 2;

    /* E2M1: 1 sign, 2 exponent bits (bias 1, field 0 subnormal), 1 mantissa bit */
    for (int i = 0; i < 8; ++i) {
        int e = i >> 1, m = i & 1;
        e2m1_grid[i] = e == 0 ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);
    }
    /* E4M3FN: codes 0..126 are the finite non-negative values (127 is NaN) */
    for (int i = 0; i < 127; ++i) {
        int e = i >> 3, m = i & 7;
        e4m3_grid[i] = e == 0 ? ldexp((double)m, -9) : ldexp(1.0 + m / 8.0, e - 7);
    }

    long long bad2 = 0, bad4 = 0, tested = 0;
    uint32_t first2 = 0, first4 = 0;
    #pragma omp parallel for reduction(+:bad2,bad4,tested) schedule(static)
    for (long long b = 0; b < (1LL << 32); ++b) {
        uint32_t bits = (uint32_t)b;
        float x;
        memcpy(&x, &bits, 4);
        if (isnan(x)) continue;
        ++tested;
        if (o_e2m1(x) != brute_e2m1(x)) { if (!bad2) first2 = bits; ++bad2; }
        if (o_e4m3(x) != brute_e4m3(x)) { if (!bad4) first4 = bits; ++bad4; }
    }
    printf("tested %lld e2m1_mismatch %lld first 0x%08x e4m3_mismatch %lld first 0x%08x\n",
           tested, bad2, first2, bad4, first4);
    return (bad2 || bad4) ? 1 : 0;
}
