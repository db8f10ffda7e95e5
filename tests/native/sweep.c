/*
 * Exhaustive checks of the oracle's E2M1 and E4M3 rounding against an
 * independent nearest-value search (test code; links the oracle library).
 *
 * The candidate grids are rebuilt here from the format definitions, not
 * taken from the oracle: E2M1 magnitudes are the code points printed in
 * "Hardware FP4 inference for speech on Blackwell", section "NVFP4, and the
 * two ways it fails"; E4M3 values come from its bit fields (bias 7, three
 * mantissa bits, largest finite 448 as stated on the same page).
 *
 * Both sweeps cover every positive finite binary32 bit pattern
 * (0x00000001 .. 0x7F7FFFFF) and, for E2M1, the negative mirror as well.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

unsigned orc_e2m1_encode(double v);
unsigned orc_e4m3_encode_satfinite(float v);

static const double kE2M1[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

static float bits_to_f32(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }

/* Nearest E2M1 magnitude index by scanning all eight candidates; an exact
 * tie goes to the even index (mantissa bit 0); anything above 6 maps to 6. */
static unsigned brute_e2m1(double a)
{
    if (a >= kE2M1[7]) return 7;          /* saturate above 6 */
    unsigned best = 0;
    double bd = fabs(a - kE2M1[0]);
    for (unsigned i = 1; i < 8; ++i) {
        double d = fabs(a - kE2M1[i]);
        if (d < bd || (d == bd && (i % 2 == 0))) { bd = d; best = i; }
    }
    return best;
}

/* Returns the number of bit patterns in [lo, hi) where the oracle differs
 * from the brute-force search, for +v and for -v.  first_bad receives the
 * first failing pattern (or 0). */
long sweep_e2m1(uint32_t lo, uint32_t hi, uint32_t* first_bad)
{
    long bad = 0;
    uint32_t fb = 0;
#pragma omp parallel for reduction(+:bad) schedule(static)
    for (int64_t u = lo; u < (int64_t)hi; ++u) {
        float v = bits_to_f32((uint32_t)u);
        unsigned want = brute_e2m1(fabs((double)v));
        unsigned got_p = orc_e2m1_encode((double)v);
        unsigned got_n = orc_e2m1_encode(-(double)v);
        if (got_p != want || got_n != (8u | want)) {
            ++bad;
#pragma omp critical
            if (fb == 0 || (uint32_t)u < fb) fb = (uint32_t)u;
        }
    }
    *first_bad = fb;
    return bad;
}

/* Sorted E4M3 finite non-negative values from the bit fields. */
static int e4m3_grid(double* val, unsigned* code)
{
    int n = 0;
    for (unsigned c = 0; c <= 0x7E; ++c) {
        unsigned e = c >> 3, m = c & 7;
        val[n] = e == 0 ? ldexp((double)m, -9) : ldexp(1.0 + m / 8.0, (int)e - 7);
        code[n] = c;
        ++n;
    }
    return n;  /* 127 values, ascending */
}

/* Nearest E4M3 value by bisection over the sorted grid, tie to the code with
 * an even mantissa, values above 448 saturate to 448. */
static unsigned brute_e4m3(double a, const double* val, const unsigned* code, int n)
{
    if (a >= val[n - 1]) return code[n - 1];
    int lo = 0, hi = n - 1;              /* val[lo] <= a < val[hi] */
    while (hi - lo > 1) {
        int mid = (lo + hi) / 2;
        if (val[mid] <= a) lo = mid; else hi = mid;
    }
    double dl = a - val[lo], dh = val[hi] - a;
    if (dl < dh) return code[lo];
    if (dh < dl) return code[hi];
    return (code[lo] % 2 == 0) ? code[lo] : code[hi];
}

long sweep_e4m3(uint32_t lo, uint32_t hi, uint32_t* first_bad)
{
    double val[128];
    unsigned code[128];
    int n = e4m3_grid(val, code);
    long bad = 0;
    uint32_t fb = 0;
#pragma omp parallel for reduction(+:bad) schedule(static)
    for (int64_t u = lo; u < (int64_t)hi; ++u) {
        float v = bits_to_f32((uint32_t)u);
        unsigned want = brute_e4m3((double)v, val, code, n);
        unsigned got = orc_e4m3_encode_satfinite(v);
        if (got != want) {
            ++bad;
#pragma omp critical
            if (fb == 0 || (uint32_t)u < fb) fb = (uint32_t)u;
        }
    }
    *first_bad = fb;
    return bad;
}
