/*
 * fp4_oracle.c -- plain CPU oracle for W4A4 block-scaled FP4 (NVFP4 / MXFP4).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may call this code:
 * only tests/, __graft_entry__.smoke() and bench.py's cpu_baseline leg (and
 * `bench.py --impl reference`) load it.  It shares no code, header, table or
 * helper with the CUDA library under mxfp4_block_scaled_fp4_b200/csrc.
 *
 * Sources (page title, section):
 *  [HW4] "Hardware FP4 inference for speech on Blackwell", section
 *        "NVFP4, and the two ways it fails": E2M1 code points, 16-value
 *        blocks with an E4M3 scale cast from max|x|/6, x_hat = s*q, E4M3
 *        maximum 448, per-tensor FP32 scale that saturates instead of NaN.
 *  [DIA] "FP4 n'existe pas : il existe des FP4, et chaque runtime choisit son
 *        dialecte", section "Deux dialectes, deux strategies de scaling" and
 *        its format table: MXFP4 = OCP MX v1.0, 32-value blocks sharing an
 *        E8M0 power-of-two exponent; NVFP4 = 16-value blocks, E4M3 scale plus
 *        an FP32 per-tensor scale; E2M1 = sign, 2 exponent bits, 1 mantissa.
 *  [5090] "FP4 on a consumer RTX 5090: the Blackwell headline loses to plain
 *        int4", section "Finding 3 -- the real-FP4 path (QuTLASS MXFP4)":
 *        every layer pays an online Hadamard rotation plus activation
 *        quantization.
 *
 * Readings where the pages leave a step open:
 *  R1 every FP32 step below is one correctly rounded IEEE binary32
 *     operation (round to nearest even), no FMA contraction; bf16 inputs are
 *     widened exactly to FP32;
 *  R2 DYNAMIC global scale g = RN(amax_t / 2688), g = 1 when amax_t == 0;
 *  R3 block scale: d = RN(6*g), sb = RN(b/d), s = E4M3 RNE with saturation
 *     to 448 ("cast" read as round-to-nearest-even, satfinite);
 *  R4 element code: r = RN(1 / RN(s*g)), v = RN(x*r), q = E2M1 RNE with
 *     saturation to 6; the sign of v is kept, so a negative v that rounds to
 *     zero gives code 0x8; a block whose scale code is 0 gets all-zero codes;
 *  R5 MXFP4 exponent e = floor(log2 b) - 2 (2 = largest E2M1 exponent),
 *     clamped to [-127, 127], e = -127 when b == 0; scale byte = e + 127;
 *     v = x * 2^-e computed exactly; q = E2M1 RNE with saturation to 6;
 *  R6 packing: element 2j goes to the low nibble of byte j of its row.
 *  R7 online rotation ([5090], section "Finding 3 -- the real-FP4 path
 *     (QuTLASS MXFP4)": an online Hadamard rotation ahead of the activation
 *     quantizer): block-diagonal Walsh-Hadamard along K, n in {16, 32}
 *     consecutive values per block from k = 0, Sylvester order
 *     H[i][j] = (-1)^popcount(i & j).  Computed in binary32 as the fast
 *     transform: for h = 1, 2, 4, ... < n, every pair (i, i + h) with bit h
 *     of i clear becomes (RN(a + b), RN(a - b)); then every value is
 *     multiplied by 2^-shift (exact: every intermediate is a multiple of the
 *     smallest bf16 step, so the scaling never rounds).  The two operands of
 *     a GEMM take shifts that add up to log2(n), so that the rotated
 *     product equals the plain one: activations ceil(log2(n)/2), weights
 *     floor(log2(n)/2).  The quantizers then take the binary32 rotated
 *     values exactly as they take widened bf16 values (R1-R5), the DYNAMIC
 *     amax included;
 *  R8 MXFP4 "overflow-aware" scale rule (OAS; [DIA], section "L'ecart de
 *     qualite -- et comment il se reduit": the block scale is chosen so
 *     that the extreme values do not saturate): e = the smallest integer
 *     with b <= 6 * 2^e, i.e. e = floor(log2 b) - 2 when b / 2^floor(log2 b)
 *     <= 1.5 and one more otherwise, clamped to [-127, 127] (-127 for a zero
 *     block).  R5 is the OCP rule, which lets values in (6, 8) * 2^e clip.
 *  R9 MXFP4 macro-block scaling (MBS; [DIA], same section: a second-level
 *     scale over a "macro-block" grouping several 32-blocks, the base
 *     format unchanged, bringing MXFP4 close to two-level scaling): the
 *     macro-block is one row (all K / 32 blocks of a token or an output
 *     channel, so that the GEMM applies the second level in its epilogue
 *     as sigma_a[m] * sigma_w[n]).  Per row: A = max |x| (exact);
 *     t = RN(A / 6); sigma = t * 2^-floor(log2 t) (exact: t's significand,
 *     in [1, 2)); sigma = 1 when A == 0; rho = RN(1 / sigma);
 *     x' = RN(x * rho); then the MXFP4 block quantizer (R5 or R8) on x'.
 *     The row's largest block then sits at the top of its E2M1 range;
 *     x_hat = sigma * 2^e * q.
 *
 * Build: gcc -O2 -fopenmp -ffp-contract=off -fno-fast-math -shared -fPIC
 * (oracle/build.py).  FP32 arithmetic is SSE binary32 on x86-64
 * (FLT_EVAL_METHOD == 0), so each float expression rounds once.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#if defined(__FLT_EVAL_METHOD__) && __FLT_EVAL_METHOD__ != 0
#error "the oracle needs binary32 evaluation of float expressions"
#endif

#define ORC_OK 0
#define ORC_BAD_SHAPE 1

/* ---------------------------------------------------------------- bf16 -- */

/* bf16 is the top half of a binary32: widening is exact. */
float orc_bf16_to_f32(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* ---------------------------------------------------------------- E2M1 -- */

/* Decode one 4-bit E2M1 code from its fields ([DIA]: sign, 2 exponent bits,
 * 1 mantissa bit; exponent bias 1, exponent field 0 is subnormal).  The
 * magnitudes must come out as the page's list {0,0.5,1,1.5,2,3,4,6} ([HW4]);
 * a test checks that. */
double orc_e2m1_decode(unsigned code)
{
    unsigned sign = (code >> 3) & 1u, ex = (code >> 1) & 3u, man = code & 1u;
    double mag = (ex == 0) ? 0.5 * man : ldexp(1.0 + 0.5 * man, (int)ex - 1);
    return sign ? -mag : mag;
}

/* The eight non-negative E2M1 magnitudes in code order (code 0..7). */
static double e2m1_mag(unsigned idx) { return orc_e2m1_decode(idx & 7u); }

/* Round a finite value to E2M1: nearest magnitude, a tie goes to the code
 * with a zero mantissa bit (even code), magnitudes above 6 saturate to 6
 * (R4).  The sign bit is copied from v, including for -0 and for negative
 * values that round to zero. */
unsigned orc_e2m1_encode(double v)
{
    unsigned sign = signbit(v) ? 8u : 0u;
    double a = fabs(v);
    unsigned idx = 7;
    for (unsigned i = 0; i < 7; ++i) {
        double lo = e2m1_mag(i), hi = e2m1_mag(i + 1);
        if (a < hi) {
            double mid = 0.5 * (lo + hi);          /* exact in binary64 */
            if (a < mid)       idx = i;
            else if (a > mid)  idx = i + 1;
            else               idx = (i % 2 == 0) ? i : i + 1;
            break;
        }
    }
    return sign | idx;
}

/* ---------------------------------------------------------------- E4M3 -- */

/* OCP E4M3 ("FN"): bias 7, 3 mantissa bits, exponent field 0 subnormal
 * (m * 2^-9), 0x7F / 0xFF are NaN, largest finite 0x7E = 448 ([HW4]). */
double orc_e4m3_decode(unsigned code)
{
    unsigned sign = (code >> 7) & 1u, ex = (code >> 3) & 15u, man = code & 7u;
    double mag;
    if (ex == 15 && man == 7) return NAN;
    if (ex == 0) mag = ldexp((double)man, -9);
    else         mag = ldexp(1.0 + man / 8.0, (int)ex - 7);
    return sign ? -mag : mag;
}

/* Round a non-negative finite binary32 to E4M3 (R3): round to nearest even
 * on the E4M3 grid, anything above 448 saturates to 448 (code 0x7E).  The
 * sign bit of the result is 0.  Steps: find the binade, take its quantum
 * (2^-9 in the subnormal range), round v/quantum to an integer with ties to
 * even, re-encode. */
unsigned orc_e4m3_encode_satfinite(float v)
{
    double x = (double)v;
    if (!(x > 0.0)) return 0u;                 /* +0, -0 (scales are |.|) */
    if (x >= 448.0) return 0x7Eu;
    int e2;
    frexp(x, &e2);                             /* x = f * 2^e2, f in [0.5,1) */
    int ex = e2 - 1;                           /* floor(log2 x) */
    if (ex < -6) ex = -6;                      /* below 2^-6: subnormal step */
    double quantum = ldexp(1.0, ex - 3);
    double n = nearbyint(x / quantum);         /* exact division; RNE */
    double r = n * quantum;
    if (r >= 464.0) return 0x7Eu;              /* cannot happen below 448 */
    if (r == 0.0) return 0u;
    if (r < ldexp(1.0, -6)) {                  /* subnormal: m * 2^-9 */
        return (unsigned)(r / ldexp(1.0, -9));
    }
    int f2;
    double fr = frexp(r, &f2);                 /* r = fr * 2^f2 */
    int eu = f2 - 1;                           /* unbiased exponent */
    unsigned man = (unsigned)((fr * 2.0 - 1.0) * 8.0);
    return ((unsigned)(eu + 7) << 3) | man;
}

/* ---------------------------------------------------------------- E8M0 -- */

/* E8M0 ([DIA]): an 8-bit biased exponent, value 2^(code-127); 0xFF is NaN. */
double orc_e8m0_decode(unsigned code)
{
    if ((code & 0xFFu) == 0xFFu) return NAN;
    return ldexp(1.0, (int)(code & 0xFFu) - 127);
}

/* ------------------------------------------------------- global scale -- */

float orc_amax_bf16(const uint16_t* x, long n)
{
    float m = 0.0f;
    for (long i = 0; i < n; ++i) {
        float a = fabsf(orc_bf16_to_f32(x[i]));
        if (a > m) m = a;
    }
    return m;
}

/* R2: g = RN(amax / 2688) with 2688 = 6 * 448; an all-zero tensor gets 1. */
float orc_nvfp4_global_scale(float amax)
{
    if (amax == 0.0f) return 1.0f;
    return amax / 2688.0f;
}

/* ----------------------------------------------------------- NVFP4 -- */

/* One NVFP4 block of 16 binary32 values ([HW4] with R3/R4; bf16 inputs are
 * widened exactly first).  Writes 16 codes (one per byte, unpacked) and
 * returns the E4M3 scale byte. */
static unsigned nvfp4_block(const float* x, float g, unsigned char q[16])
{
    float b = 0.0f;
    for (int i = 0; i < 16; ++i) {
        float a = fabsf(x[i]);
        if (a > b) b = a;
    }
    float d = 6.0f * g;
    float sb = b / d;
    unsigned s = orc_e4m3_encode_satfinite(sb);
    float sv = (float)orc_e4m3_decode(s);      /* exact: E4M3 fits binary32 */
    if (sv == 0.0f) {
        for (int i = 0; i < 16; ++i) q[i] = 0;
        return s;
    }
    float sg = sv * g;
    float r = 1.0f / sg;
    for (int i = 0; i < 16; ++i) {
        float v = x[i] * r;
        q[i] = (unsigned char)orc_e2m1_encode((double)v);
    }
    return s;
}

/* amax over a binary32 tensor (exact). */
float orc_amax_f32(const float* x, long n)
{
    float m = 0.0f;
    for (long i = 0; i < n; ++i) {
        float a = fabsf(x[i]);
        if (a > m) m = a;
    }
    return m;
}

/* NVFP4 of a row-major binary32 [rows, K] tensor; g as for the bf16 form. */
int orc_nvfp4_quantize_f32(const float* x, long rows, long K, int dynamic,
                           float* g, uint8_t* codes, uint8_t* scales)
{
    if (rows < 0 || K <= 0 || K % 16 != 0) return ORC_BAD_SHAPE;
    if (dynamic) *g = orc_nvfp4_global_scale(orc_amax_f32(x, rows * K));
    const float gg = *g;
    const long nb = K / 16;
#pragma omp parallel for schedule(static)
    for (long r = 0; r < rows; ++r) {
        for (long b = 0; b < nb; ++b) {
            unsigned char q[16];
            scales[r * nb + b] =
                (uint8_t)nvfp4_block(x + r * K + b * 16, gg, q);
            for (int j = 0; j < 8; ++j)
                codes[r * (K / 2) + b * 8 + j] =
                    (uint8_t)(q[2 * j] | (q[2 * j + 1] << 4));
        }
    }
    return ORC_OK;
}

/* Quantize a row-major bf16 [rows, K] tensor to NVFP4.
 *   dynamic != 0 : *g is written with R2's value from the tensor's amax;
 *   dynamic == 0 : *g is read (a caller-chosen global scale; 1 = none).
 * codes:  [rows, K/2] bytes, two codes per byte (R6).
 * scales: [rows, K/16] E4M3 bytes, row-major (canonical order). */
int orc_nvfp4_quantize(const uint16_t* x, long rows, long K, int dynamic,
                       float* g, uint8_t* codes, uint8_t* scales)
{
    if (rows < 0 || K <= 0 || K % 16 != 0) return ORC_BAD_SHAPE;
    if (dynamic) *g = orc_nvfp4_global_scale(orc_amax_bf16(x, rows * K));
    const float gg = *g;
    const long nb = K / 16;
#pragma omp parallel for schedule(static)
    for (long r = 0; r < rows; ++r) {
        for (long b = 0; b < nb; ++b) {
            float xf[16];
            unsigned char q[16];
            for (int i = 0; i < 16; ++i)
                xf[i] = orc_bf16_to_f32(x[r * K + b * 16 + i]);
            scales[r * nb + b] = (uint8_t)nvfp4_block(xf, gg, q);
            for (int j = 0; j < 8; ++j)
                codes[r * (K / 2) + b * 8 + j] =
                    (uint8_t)(q[2 * j] | (q[2 * j + 1] << 4));
        }
    }
    return ORC_OK;
}

/* ----------------------------------------------------------- MXFP4 -- */

/* floor(log2(a)) of a positive finite binary32, read from its bits. */
static int floor_log2_f32(float a)
{
    uint32_t u;
    memcpy(&u, &a, sizeof u);
    int ex = (int)((u >> 23) & 0xFFu);
    uint32_t man = u & 0x7FFFFFu;
    if (ex != 0) return ex - 127;
    /* subnormal: value = man * 2^-149 */
    int msb = 31 - __builtin_clz(man);
    return msb - 149;
}

/* The MXFP4 block exponent of a block maximum b >= 0: rule 0 is R5 (OCP,
 * floor(log2 b) - 2), rule 1 is R8 (OAS: the smallest e with b <= 6 * 2^e).
 * Clamped to [-127, 127]; -127 for b == 0. */
static int mxfp4_exponent(float b, int rule)
{
    if (b == 0.0f) return -127;
    int e = floor_log2_f32(b) - 2;
    if (rule == 1 && (double)b > ldexp(6.0, e)) e += 1;   /* exact comparison */
    if (e < -127) e = -127;
    if (e > 127) e = 127;
    return e;
}

/* One MXFP4 block of 32 binary32 values (R5 / R8).  Returns the E8M0 scale
 * byte. */
static unsigned mxfp4_block(const float* x, int rule, unsigned char q[32])
{
    float b = 0.0f;
    for (int i = 0; i < 32; ++i) {
        float a = fabsf(x[i]);
        if (a > b) b = a;
    }
    int e = mxfp4_exponent(b, rule);
    for (int i = 0; i < 32; ++i) {
        double v = ldexp((double)x[i], -e);   /* exact */
        q[i] = (unsigned char)orc_e2m1_encode(v);
    }
    return (unsigned)(e + 127);
}

/* MXFP4 of a row-major binary32 [rows, K] tensor with scale rule `rule`
 * (0 = OCP R5, 1 = OAS R8). */
int orc_mxfp4_quantize_f32(const float* x, long rows, long K, int rule,
                           uint8_t* codes, uint8_t* scales)
{
    if (rows < 0 || K <= 0 || K % 32 != 0 || rule < 0 || rule > 1) return ORC_BAD_SHAPE;
    const long nb = K / 32;
#pragma omp parallel for schedule(static)
    for (long r = 0; r < rows; ++r) {
        for (long b = 0; b < nb; ++b) {
            unsigned char q[32];
            scales[r * nb + b] = (uint8_t)mxfp4_block(x + r * K + b * 32, rule, q);
            for (int j = 0; j < 16; ++j)
                codes[r * (K / 2) + b * 16 + j] =
                    (uint8_t)(q[2 * j] | (q[2 * j + 1] << 4));
        }
    }
    return ORC_OK;
}

/* Quantize a row-major bf16 [rows, K] tensor to MXFP4 (no global scale),
 * OCP rule (R5).  codes: [rows, K/2]; scales: [rows, K/32] E8M0 bytes,
 * row-major. */
int orc_mxfp4_quantize(const uint16_t* x, long rows, long K,
                       uint8_t* codes, uint8_t* scales)
{
    if (rows < 0 || K <= 0 || K % 32 != 0) return ORC_BAD_SHAPE;
    const long nb = K / 32;
#pragma omp parallel for schedule(static)
    for (long r = 0; r < rows; ++r) {
        for (long b = 0; b < nb; ++b) {
            float xf[32];
            unsigned char q[32];
            for (int i = 0; i < 32; ++i)
                xf[i] = orc_bf16_to_f32(x[r * K + b * 32 + i]);
            scales[r * nb + b] = (uint8_t)mxfp4_block(xf, 0, q);
            for (int j = 0; j < 16; ++j)
                codes[r * (K / 2) + b * 16 + j] =
                    (uint8_t)(q[2 * j] | (q[2 * j + 1] << 4));
        }
    }
    return ORC_OK;
}

/* ------------------------------------------ macro-block scaling (R9) -- */

/* The macro scale of a row from its largest magnitude A (R9). */
float orc_mbs_sigma(float A)
{
    if (A == 0.0f) return 1.0f;
    float t = A / 6.0f;
    int ex = floor_log2_f32(t);
    return (float)ldexp((double)t, -ex);       /* exact: t's significand */
}

/* MXFP4 with a macro scale per row (R9): sigma[rows] out, codes
 * [rows, K/2], scales [rows, K/32] (rule as in orc_mxfp4_quantize_f32). */
int orc_mxfp4_mbs_quantize(const uint16_t* x, long rows, long K, int rule,
                           float* sigma, uint8_t* codes, uint8_t* scales)
{
    if (rows < 0 || K <= 0 || K % 32 != 0 || rule < 0 || rule > 1) return ORC_BAD_SHAPE;
    const long nb = K / 32;
#pragma omp parallel for schedule(static)
    for (long r = 0; r < rows; ++r) {
        float A = 0.0f;
        for (long k = 0; k < K; ++k) {
            float a = fabsf(orc_bf16_to_f32(x[r * K + k]));
            if (a > A) A = a;
        }
        const float sg = orc_mbs_sigma(A);
        const float rho = 1.0f / sg;
        sigma[r] = sg;
        for (long b = 0; b < nb; ++b) {
            float xf[32];
            unsigned char q[32];
            for (int i = 0; i < 32; ++i)
                xf[i] = orc_bf16_to_f32(x[r * K + b * 32 + i]) * rho;
            scales[r * nb + b] = (uint8_t)mxfp4_block(xf, rule, q);
            for (int j = 0; j < 16; ++j)
                codes[r * (K / 2) + b * 16 + j] =
                    (uint8_t)(q[2 * j] | (q[2 * j + 1] << 4));
        }
    }
    return ORC_OK;
}

/* ------------------------------------------------- online rotation (R7) -- */

/* Rotate every n-value block of every row of a bf16 [rows, K] tensor by the
 * Walsh-Hadamard matrix of order n (n = 16 or 32, K % n == 0), in binary32
 * by the fast transform of R7, then scale by 2^-shift (0 <= shift <= 8).
 * out: binary32 [rows, K]. */
int orc_hadamard_f32(const uint16_t* x, long rows, long K, int n, int shift,
                     float* out)
{
    if (rows < 0 || K <= 0 || (n != 16 && n != 32) || K % n != 0 ||
        shift < 0 || shift > 8)
        return ORC_BAD_SHAPE;
    const float scale = ldexpf(1.0f, -shift);
#pragma omp parallel for schedule(static)
    for (long r = 0; r < rows; ++r) {
        for (long b = 0; b < K / n; ++b) {
            float v[32];
            for (int i = 0; i < n; ++i) v[i] = orc_bf16_to_f32(x[r * K + b * n + i]);
            for (int h = 1; h < n; h *= 2)
                for (int i = 0; i < n; ++i)
                    if ((i & h) == 0) {
                        float a = v[i], c = v[i + h];
                        v[i] = a + c;
                        v[i + h] = a - c;
                    }
            for (int i = 0; i < n; ++i) out[r * K + b * n + i] = v[i] * scale;
        }
    }
    return ORC_OK;
}

/* ----------------------------------------------------------- dequant -- */

/* x_hat = g * s * q in binary64 (every factor and product is exact).
 * fmt 0 = NVFP4 (16-blocks, E4M3 scales, global g); 1 = MXFP4 (32-blocks,
 * E8M0 scales, g ignored).  Scales in row-major canonical order. */
int orc_dequant(const uint8_t* codes, const uint8_t* scales, long rows, long K,
                int fmt, float g, double* out)
{
    const long bs = fmt == 0 ? 16 : 32;
    if (K % bs != 0) return ORC_BAD_SHAPE;
    const long nb = K / bs;
#pragma omp parallel for schedule(static)
    for (long r = 0; r < rows; ++r) {
        for (long k = 0; k < K; ++k) {
            uint8_t byte = codes[r * (K / 2) + k / 2];
            unsigned c = (k % 2 == 0) ? (byte & 15u) : (byte >> 4);
            uint8_t sc = scales[r * nb + k / bs];
            double s = fmt == 0 ? (double)g * orc_e4m3_decode(sc)
                                : orc_e8m0_decode(sc);
            out[r * K + k] = s * orc_e2m1_decode(c);
        }
    }
    return ORC_OK;
}

/* ------------------------------------------------------------- GEMM -- */

/* C[m,n] = sum_k A[m,k] * W[n,k], the plain triple loop in binary64. */
void orc_gemm_naive(const double* A, const double* W, long M, long N, long K,
                    double* C)
{
#pragma omp parallel for schedule(static)
    for (long m = 0; m < M; ++m)
        for (long n = 0; n < N; ++n) {
            double acc = 0.0;
            for (long k = 0; k < K; ++k) acc += A[m * K + k] * W[n * K + k];
            C[m * N + n] = acc;
        }
}

/* ------------------------------------------ MMA-consumable scale order -- */

/* The scale layout the block-scaled tensor-core MMA reads (a reading: the
 * pages do not describe it).  Scales are grouped in atoms of 128 rows x 4
 * scale columns (512 bytes).  Inside an atom, row r and column c sit at
 * byte (r % 32) * 16 + (r / 32) * 4 + c.  Atoms are stored with the scale-
 * column group fastest: atom (rb, cb) starts at (rb * ncb + cb) * 512, with
 * ncb = ceil(nsf / 4).  Rows are padded to a multiple of 128 and columns to
 * a multiple of 4; padding bytes are 0. */
long orc_mma_scale_bytes(long rows, long nsf)
{
    long rb = (rows + 127) / 128, cb = (nsf + 3) / 4;
    return rb * cb * 512;
}

long orc_mma_scale_offset(long r, long c, long nsf)
{
    long ncb = (nsf + 3) / 4;
    long atom = (r / 128) * ncb + c / 4;
    long rr = r % 128;
    return atom * 512 + (rr % 32) * 16 + (rr / 32) * 4 + (c % 4);
}

void orc_scales_to_mma(const uint8_t* rowmajor, long rows, long nsf,
                       uint8_t* mma)
{
    memset(mma, 0, (size_t)orc_mma_scale_bytes(rows, nsf));
    for (long r = 0; r < rows; ++r)
        for (long c = 0; c < nsf; ++c)
            mma[orc_mma_scale_offset(r, c, nsf)] = rowmajor[r * nsf + c];
}

void orc_scales_from_mma(const uint8_t* mma, long rows, long nsf,
                         uint8_t* rowmajor)
{
    for (long r = 0; r < rows; ++r)
        for (long c = 0; c < nsf; ++c)
            rowmajor[r * nsf + c] = mma[orc_mma_scale_offset(r, c, nsf)];
}

/* ------------------------------------------------- array conveniences -- */

void orc_e2m1_encode_array(const double* v, long n, uint8_t* out)
{
    for (long i = 0; i < n; ++i) out[i] = (uint8_t)orc_e2m1_encode(v[i]);
}

void orc_e4m3_encode_array(const float* v, long n, uint8_t* out)
{
    for (long i = 0; i < n; ++i)
        out[i] = (uint8_t)orc_e4m3_encode_satfinite(v[i]);
}
