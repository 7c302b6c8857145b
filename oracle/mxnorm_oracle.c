/*
 * mxnorm_oracle.c -- plain, slow CPU oracle for MXNorm and its companions.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test-suite, the smoke check and the
 * benchmark's CPU-baseline leg load this file's library.  It shares no code,
 * header, table or constant generator with the CUDA library; neither side
 * includes or links the other.
 *
 * What it follows (each function names its passage again):
 *  [MX]  gist.science, "MXNorm: Reusing MXFP block scales for efficient tensor
 *        normalisation", technical summary section 2.1: split each row into
 *        K = D/B blocks (B = 32), take each block's absolute maximum m_k, form
 *        the generalised p-mean G = ((1/K) sum_k m_k^p)^(1/p) as the RMS
 *        estimate, normalise by it and cast to MX in the same pass.
 *        Section 2.2: RMSNorm output bounded by sqrt(D), MXNorm's by a bound in K.
 *        Section 2.3: gamma may be folded into the next weight; the backward
 *        reuses the RMSNorm gradient as a straight-through estimator.
 *        Section 1.2: RMSNorm then MXCast as two separate steps (the baseline).
 *  [RC]  fugumt, "Recipes for Pre-training LLMs with MXFP8", abstract:
 *        MXFP8-E4M3 with a specific conversion algorithm.  Reading adopted:
 *        the E8M0 scale is the smallest power of two 2^e for which the block
 *        absmax does not exceed the E4M3 maximum, i.e. no element saturates.
 *  [F8]  "FP8 Formats for Deep Learning" (listed on the same page): E4M3 has
 *        no infinities and one NaN mantissa pattern, so its largest finite
 *        value is 448 = 1.75 * 2^8; exponent bias 7, subnormal step 2^-9.
 *  [SR]  aibr.jp article on stochastic rounding with BF16 and Adam, section 3:
 *        round to one of the two neighbouring representable values, with
 *        probability set by the distance, so the expectation equals the input.
 *  [PX]  Philox4x32-10: Salmon, Moraes, Dror, Shaw, "Parallel random numbers:
 *        as easy as 1, 2, 3", SC'11 (multipliers, Weyl key increments, round
 *        function S-box as published there).
 *  [F4]  The FP4 variant the MXNorm summary reports a layer speedup for
 *        (section 3, "NVFP4"; the related-papers lists on the same pages train
 *        in FP4).  The pages do not define the element format; the reading
 *        adopted is the E2M1 element of the OCP Microscaling (MX) v1.0 format
 *        (1 sign, 2 exponent bits with bias 1, 1 mantissa bit, no infinity or
 *        NaN: magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6) in blocks of 32 with one
 *        E8M0 scale (MXFP4), the scale rounded up as in [RC] with 6 in place
 *        of 448.
 *  [SE]  Scale reuse (the MXNorm title: reusing the block scales): the block
 *        statistic m_k replaced by the block's own power-of-two scale 2^e_k,
 *        e_k the [RC] exponent of m_k.
 *  [NV]  NVFP4, the FP4 format the MXNorm summary (section 3) reports its
 *        layer speedup with; the pages name it without defining it.  Reading
 *        adopted: E2M1 elements [F4] in blocks of 16, each block with a
 *        positive E4M3 scale [F8], the smallest E4M3 value s with
 *        amax <= 6 s (rounded up, as [RC]), and no tensor-wide scale (MXNorm
 *        already bounds |y| by K^(1/p) max|gamma|, so the scales stay inside
 *        E4M3's range); codes E2M1(fl32(y * fl32(1/s))).  The MXNorm statistic
 *        then runs over the 16-element blocks.
 *
 * Precision: statistics (G, RMS, backward sums) in long double / double.
 * Where floating point decides an integer code, the oracle takes that decision
 * in the precision the kernel uses (fp32, IEEE round-to-nearest-even, no
 * flush-to-zero): s = fl32(1/G), y = fl32(fl32(x*s)*gamma), v = fl32(y*2^-e).
 * Build with -ffp-contract=off and without -ffast-math so that each of those
 * is one correctly rounded fp32 operation.
 */
#include <float.h>
#include <math.h>
#include <stdint.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_BLOCK 32          /* MX block size B [MX 2.1] */
#define E4M3_MAX 448.0           /* [F8] */
#define E2M1_MAX 6.0             /* [F4] */
#define ORACLE_FMT_E4M3 0
#define ORACLE_FMT_E2M1 1
#define ORACLE_FMT_NVFP4 2
#define NVFP4_BLOCK 16           /* [NV] */

/* ---------------------------------------------------------------- helpers */

static float bf16_to_f32(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

static uint32_t f32_bits(float f)
{
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    return u;
}

/* Round a double to the nearest bf16 (ties to even), once. */
static uint16_t bf16_rne_from_double(double v)
{
    if (isnan(v)) return 0x7FC0;
    uint16_t sign = signbit(v) ? 0x8000 : 0;
    double a = fabs(v);
    if (a == 0.0) return sign;
    int E;
    frexp(a, &E);                     /* a = f * 2^E, f in [0.5, 1) */
    int b = E - 1;                    /* a in [2^b, 2^(b+1)) */
    if (b < -126) b = -126;           /* subnormal bf16: fixed spacing 2^-133 */
    double step = ldexp(1.0, b - 7);  /* bf16 keeps 7 fraction bits */
    double n = a / step;              /* exact: division by a power of two */
    double k = floor(n), rem = n - k;
    if (rem > 0.5 || (rem == 0.5 && fmod(k, 2.0) == 1.0)) k += 1.0;
    double r = k * step;
    if (r > 0x1.FEp127) return sign | 0x7F80;  /* overflow to infinity */
    float rf = (float)r;              /* exact: r is a bf16 value */
    return sign | (uint16_t)(f32_bits(rf) >> 16);
}

/* ------------------------------------------------------------ E4M3 [F8] */

/* Value of a non-negative E4M3 code c in [0, 0x7E]. */
double oracle_e4m3_value(int c)
{
    int ex = (c >> 3) & 15, man = c & 7;
    if (ex == 0) return ldexp((double)man, -9);      /* subnormal: man * 2^-9 */
    return ldexp(1.0 + man / 8.0, ex - 7);           /* (1 + man/8) * 2^(ex-7) */
}

/* Spacing of the E4M3 grid around a magnitude a < 448. */
static double e4m3_step(double a)
{
    if (a < 0x1p-6) return 0x1p-9;    /* below the smallest normal: subnormal step */
    int E;
    frexp(a, &E);
    return ldexp(1.0, (E - 1) - 3);   /* 3 fraction bits in binade [2^(E-1), 2^E) */
}

/* Code of a non-negative grid value r (0 <= r <= 448). */
static uint8_t e4m3_encode_grid(double r)
{
    if (r < 0x1p-6) return (uint8_t)(r / 0x1p-9);          /* subnormal: r = man * 2^-9 */
    int E;
    double f = frexp(r, &E);                               /* r = f * 2^E */
    int b = E - 1;                                         /* r = (2f) * 2^b, 2f in [1,2) */
    int man = (int)((2.0 * f - 1.0) * 8.0);
    return (uint8_t)(((b + 7) << 3) | man);
}

/* fp32 -> E4M3, round to nearest, ties to even, saturating to +-448; NaN -> NaN.
   The sign bit of the input is kept (a negative value that rounds to zero
   gives 0x80). */
uint8_t oracle_e4m3_rne(float v)
{
    uint8_t sign = signbit(v) ? 0x80 : 0x00;
    if (isnan(v)) return sign | 0x7F;
    double a = fabs((double)v);
    if (a >= E4M3_MAX) return sign | 0x7E;                 /* satfinite */
    double step = e4m3_step(a);
    double n = a / step;                                   /* exact */
    double k = floor(n), rem = n - k;
    if (rem > 0.5 || (rem == 0.5 && fmod(k, 2.0) == 1.0)) k += 1.0;
    return sign | e4m3_encode_grid(k * step);
}

/* fp32 -> E4M3 by stochastic rounding [SR]: with lo <= |v| < hi the two
   neighbouring grid values, pick hi iff r32 < frac * 2^32 where
   frac = (|v| - lo) / (hi - lo).  Every quantity is exact in double. */
uint8_t oracle_e4m3_sr(float v, uint32_t r32)
{
    uint8_t sign = signbit(v) ? 0x80 : 0x00;
    if (isnan(v)) return sign | 0x7F;
    double a = fabs((double)v);
    if (a >= E4M3_MAX) return sign | 0x7E;
    double step = e4m3_step(a);
    double lo = floor(a / step) * step;
    double hi = lo + step;
    double frac = (a - lo) / (hi - lo);
    double r = ((double)r32 < frac * 4294967296.0) ? hi : lo;
    return sign | e4m3_encode_grid(r);
}

/* ------------------------------------------------------------ E2M1 [F4] */

/* Value of a non-negative E2M1 code c in [0, 7]. */
double oracle_e2m1_value(int c)
{
    int ex = (c >> 1) & 3, man = c & 1;
    if (ex == 0) return 0.5 * man;                   /* subnormal: man * 2^-1 */
    return ldexp(1.0 + man / 2.0, ex - 1);           /* (1 + man/2) * 2^(ex-1) */
}

/* Spacing of the E2M1 grid around a magnitude a < 6. */
static double e2m1_step(double a)
{
    if (a < 1.0) return 0.5;          /* below the smallest normal: subnormal step */
    int E;
    frexp(a, &E);
    return ldexp(1.0, (E - 1) - 1);   /* 1 fraction bit in binade [2^(E-1), 2^E) */
}

/* Code of a non-negative grid value r (0 <= r <= 6). */
static uint8_t e2m1_encode_grid(double r)
{
    if (r < 1.0) return (uint8_t)(r / 0.5);
    int E;
    double f = frexp(r, &E);
    int b = E - 1;
    int man = (int)((2.0 * f - 1.0) * 2.0);
    return (uint8_t)(((b + 1) << 1) | man);
}

/* fp32 -> E2M1 (4-bit code, sign in bit 3), round to nearest, ties to the
   even code, saturating to +-6.  E2M1 has no NaN: a NaN gives the saturated
   magnitude with its sign bit (the MX row code never passes one here). */
uint8_t oracle_e2m1_rne(float v)
{
    uint8_t sign = signbit(v) ? 0x8 : 0x0;
    if (isnan(v)) return sign | 0x7;
    double a = fabs((double)v);
    if (a >= E2M1_MAX) return sign | 0x7;
    double step = e2m1_step(a);
    double n = a / step;
    double k = floor(n), rem = n - k;
    if (rem > 0.5 || (rem == 0.5 && fmod(k, 2.0) == 1.0)) k += 1.0;
    return sign | e2m1_encode_grid(k * step);
}

/* fp32 -> E2M1 by stochastic rounding [SR], as oracle_e4m3_sr on the E2M1 grid. */
uint8_t oracle_e2m1_sr(float v, uint32_t r32)
{
    uint8_t sign = signbit(v) ? 0x8 : 0x0;
    if (isnan(v)) return sign | 0x7;
    double a = fabs((double)v);
    if (a >= E2M1_MAX) return sign | 0x7;
    double step = e2m1_step(a);
    double lo = floor(a / step) * step;
    double hi = lo + step;
    double frac = (a - lo) / (hi - lo);
    double r = ((double)r32 < frac * 4294967296.0) ? hi : lo;
    return sign | e2m1_encode_grid(r);
}

/* ---------------------------------------------------------- E8M0 [RC] */

/* Smallest integer e in [-127, 127] with a <= 448 * 2^e ("scale rounded up so
   that no element saturates").  Returns 128 for a NaN or infinite a. */
int oracle_e8m0_exponent(double a)
{
    if (!(a <= DBL_MAX)) return 128;
    for (int e = -127; e <= 127; ++e)
        if (a <= ldexp(E4M3_MAX, e)) return e;
    return 128;
}

/* The same rule for an element format whose largest magnitude is elem_max
   [RC][F4]: smallest e in [-127, 127] with a <= elem_max * 2^e. */
int oracle_mx_exponent(double a, double elem_max)
{
    if (!(a <= DBL_MAX)) return 128;
    for (int e = -127; e <= 127; ++e)
        if (a <= ldexp(elem_max, e)) return e;
    return 128;
}

static uint8_t e8m0_code(int e) { return e == 128 ? 0xFF : (uint8_t)(e + 127); }

/* ------------------------------------------------------ Philox4x32-10 [PX] */

void oracle_philox4x32_10(const uint32_t ctr_in[4], const uint32_t key_in[2], uint32_t out[4])
{
    const uint32_t M0 = 0xD2511F53u, M1 = 0xCD9E8D57u;   /* round multipliers */
    const uint32_t W0 = 0x9E3779B9u, W1 = 0xBB67AE85u;   /* key increments */
    uint32_t c0 = ctr_in[0], c1 = ctr_in[1], c2 = ctr_in[2], c3 = ctr_in[3];
    uint32_t k0 = key_in[0], k1 = key_in[1];
    for (int round = 0; round < 10; ++round) {
        if (round > 0) { k0 += W0; k1 += W1; }
        uint64_t p0 = (uint64_t)M0 * c0, p1 = (uint64_t)M1 * c2;
        uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
        uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
        uint32_t n0 = hi1 ^ c1 ^ k0, n1 = lo1, n2 = hi0 ^ c3 ^ k1, n3 = lo0;
        c0 = n0; c1 = n1; c2 = n2; c3 = n3;
    }
    out[0] = c0; out[1] = c1; out[2] = c2; out[3] = c3;
}

/* The random word an element draws: element index idx = row * D + col (the
   logical index, independent of the row stride); counter = (idx >> 2 as a
   64-bit number split low/high, 0, 0); key = seed split low/high; the element
   takes word idx & 3 of the four outputs. */
static uint32_t sr_word(uint64_t seed, uint64_t idx)
{
    uint64_t c = idx >> 2;
    uint32_t ctr[4] = {(uint32_t)c, (uint32_t)(c >> 32), 0u, 0u};
    uint32_t key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32)};
    uint32_t out[4];
    oracle_philox4x32_10(ctr, key, out);
    return out[idx & 3];
}

uint32_t oracle_sr_word(uint64_t seed, uint64_t idx) { return sr_word(seed, idx); }

/* -------------------------------------------------------- p-mean [MX 2.1] */

/* G = ((1/K) sum_k m_k^p)^(1/p); p = +inf gives max_k m_k.  long double keeps
   m^p finite for every finite bf16 m and p up to ~100. */
static long double pmean(const double *m, int64_t K, double p)
{
    if (isinf(p)) {
        double mx = 0.0;
        for (int64_t k = 0; k < K; ++k) if (isnan(m[k]) || m[k] > mx) mx = m[k];
        return mx;
    }
    long double s = 0.0L;
    for (int64_t k = 0; k < K; ++k) s += powl((long double)m[k], (long double)p);
    return powl(s / (long double)K, 1.0L / (long double)p);
}

double oracle_pmean(const double *m, int64_t K, double p) { return (double)pmean(m, K, p); }

/* ------------------------------------------- one row of MX quantisation */

/* Quantise one row y[0..D) (fp32 values) to MX codes + E8M0 scales [RC].
   fmt: ORACLE_FMT_E4M3 [F8] (one byte per code) or ORACLE_FMT_E2M1 [F4] (two
   codes per byte, the even column in the low nibble; D/2 bytes per row).
   rounding: 0 = nearest-even, 1 = stochastic with Philox words.
   A block holding an infinity or a NaN (outside the method's contract) gets
   the NaN scale 0xFF and a fixed code for every element (E4M3: the positive
   NaN 0x7F, the sign of a NaN made by 0 * inf differing between platforms;
   E2M1, which has no NaN: 0x7). */
static void mx_quantise_row(const float *y, int64_t D, uint8_t *q, uint8_t *scales,
                            int rounding, uint64_t seed, uint64_t row, int fmt)
{
    int64_t K = D / ORACLE_BLOCK;
    const int fp4 = (fmt == ORACLE_FMT_E2M1);
    if (fp4) memset(q, 0, (size_t)(D / 2));
    for (int64_t k = 0; k < K; ++k) {
        const float *yb = y + k * ORACLE_BLOCK;
        double a = 0.0;                                   /* block absmax of y */
        int nonfinite = 0;
        for (int i = 0; i < ORACLE_BLOCK; ++i) {
            double v = fabs((double)yb[i]);
            if (!(v <= DBL_MAX)) nonfinite = 1;
            else if (v > a) a = v;
        }
        int e = nonfinite ? 128 : (fp4 ? oracle_mx_exponent(a, E2M1_MAX) : oracle_e8m0_exponent(a));
        scales[k] = e8m0_code(e);
        for (int i = 0; i < ORACLE_BLOCK; ++i) {
            int64_t col = k * ORACLE_BLOCK + i;
            uint8_t c;
            if (e == 128) {
                c = fp4 ? 0x7 : 0x7F;                     /* non-finite block */
            } else {
                float inv_scale = ldexpf(1.0f, -e);       /* 2^-e, exact in fp32 */
                float v = yb[i] * inv_scale;              /* fp32 product, as the kernel */
                uint32_t r32 = rounding ? sr_word(seed, row * (uint64_t)D + (uint64_t)col) : 0u;
                if (fp4) c = rounding ? oracle_e2m1_sr(v, r32) : oracle_e2m1_rne(v);
                else c = rounding ? oracle_e4m3_sr(v, r32) : oracle_e4m3_rne(v);
            }
            if (fp4) q[col / 2] |= (uint8_t)(c << (4 * (col & 1)));
            else q[col] = c;
        }
    }
}

/* The NVFP4 block scale [NV]: the E4M3 code of the smallest E4M3 value s with
   a <= 6 * s (6 * s is exact in double); 0x7E (448) if none, 0 for a = 0. */
int oracle_nvfp4_scale_code(double a)
{
    for (int c = 0; c <= 0x7E; ++c)
        if (a <= 6.0 * oracle_e4m3_value(c)) return c;
    return 0x7E;
}

/* Quantise one row y[0..D) to NVFP4 [NV]: per block of 16, the E4M3 scale
   code (scales[k]) and the E2M1 codes of fl32(y * fl32(1/s)), two per byte,
   even column in the low nibble.  A zero scale (an all-zero block) gives
   zero codes; a block holding an infinity or a NaN gets the E4M3 NaN scale
   0x7F and element code 0x7. */
static void nvfp4_quantise_row(const float *y, int64_t D, uint8_t *q, uint8_t *scales,
                               int rounding, uint64_t seed, uint64_t row)
{
    int64_t K = D / NVFP4_BLOCK;
    memset(q, 0, (size_t)(D / 2));
    for (int64_t k = 0; k < K; ++k) {
        const float *yb = y + k * NVFP4_BLOCK;
        double a = 0.0;
        int nonfinite = 0;
        for (int i = 0; i < NVFP4_BLOCK; ++i) {
            double v = fabs((double)yb[i]);
            if (!(v <= DBL_MAX)) nonfinite = 1;
            else if (v > a) a = v;
        }
        int sc = nonfinite ? 0x7F : oracle_nvfp4_scale_code(a);
        scales[k] = (uint8_t)sc;
        float sval = (float)oracle_e4m3_value(sc & 0x7F);
        float inv = (sc == 0 || nonfinite) ? 0.0f : 1.0f / sval;   /* fl32(1/s) */
        for (int i = 0; i < NVFP4_BLOCK; ++i) {
            int64_t col = k * NVFP4_BLOCK + i;
            uint8_t c;
            if (nonfinite) {
                c = 0x7;
            } else if (sc == 0) {
                c = 0;
            } else {
                float v = yb[i] * inv;
                c = rounding ? oracle_e2m1_sr(v, sr_word(seed, row * (uint64_t)D + (uint64_t)col))
                             : oracle_e2m1_rne(v);
            }
            q[col / 2] |= (uint8_t)(c << (4 * (col & 1)));
        }
    }
}

static const uint16_t *row_ptr(const uint16_t *base, int64_t ld, int64_t r) { return base + r * ld; }

static int64_t pick_row(const int64_t *row_ids, int64_t i) { return row_ids ? row_ids[i] : i; }

/* ------------------------------------------------- MXNorm forward [MX 2.1] */

/*
 * For each selected row r (row_ids[i], or i when row_ids is NULL):
 *   m_k   = max_{i in block k} |x_i|                       (exact)
 *   stat = 1 [SE]: m_k <- 2^e_k, e_k the E8M0 exponent of m_k for the element
 *          format (non-finite m_k kept)
 *   G     = p-mean of m_k, in long double, rounded to fp32 -> G_out[i]
 *   if G_in is given, G_in[i] replaces G below (two-stage parity: the codes are
 *   re-derived from the kernel's G bits)
 *   s     = fl32(1/G)   (s = 0 when G = 0)
 *   y_j   = fl32(x_j * s), then y_j = fl32(y_j * gamma_j) when gamma is given
 *   scales/codes of y as in mx_quantise_row (fmt: E4M3 or E2M1).
 * Outputs are compact: q[i*D + j] (E2M1: q[i*D/2 + j/2]), scales[i*K + k], G_out[i].
 */
int oracle_mxnorm_fwd_ex(const uint16_t *x, int64_t ld_x, const uint16_t *gamma,
                         int64_t n_rows, const int64_t *row_ids, int64_t D, double p,
                         const float *G_in, uint8_t *q, uint8_t *scales, float *G_out,
                         int rounding, uint64_t seed, int stat, int fmt, int nthreads)
{
    if (D <= 0 || D % ORACLE_BLOCK != 0 || !(p > 0.0)) return -1;
    if (fmt != ORACLE_FMT_E4M3 && fmt != ORACLE_FMT_E2M1 && fmt != ORACLE_FMT_NVFP4) return -1;
    const int B = (fmt == ORACLE_FMT_NVFP4) ? NVFP4_BLOCK : ORACLE_BLOCK;   /* statistic blocks */
    int64_t K = D / B;
    const int64_t qrow = (fmt == ORACLE_FMT_E4M3) ? D : D / 2;
    const double elem_max = (fmt == ORACLE_FMT_E2M1) ? E2M1_MAX : E4M3_MAX;
#ifdef _OPENMP
    if (nthreads <= 0) nthreads = omp_get_max_threads();
#pragma omp parallel for schedule(dynamic, 4) num_threads(nthreads)
#endif
    for (int64_t i = 0; i < n_rows; ++i) {
        int64_t r = pick_row(row_ids, i);
        const uint16_t *xr = row_ptr(x, ld_x, r);
        double m[K];
        float y[D];
        for (int64_t k = 0; k < K; ++k) {
            double mk = 0.0;
            for (int j = 0; j < B; ++j) {
                double v = fabs((double)bf16_to_f32(xr[k * B + j]));
                if (isnan(v) || v > mk) mk = v;   /* a NaN, once seen, stays the max */
            }
            if (stat == 1 && mk <= DBL_MAX) {
                if (fmt == ORACLE_FMT_NVFP4) mk = oracle_e4m3_value(oracle_nvfp4_scale_code(mk));
                else mk = ldexp(1.0, oracle_mx_exponent(mk, elem_max));
            }
            m[k] = mk;
        }
        float G_ref = (float)pmean(m, K, p);
        if (G_out) G_out[i] = G_ref;
        float G = G_in ? G_in[i] : G_ref;
        float s = (G == 0.0f) ? 0.0f : 1.0f / G;
        for (int64_t j = 0; j < D; ++j) {
            float t = bf16_to_f32(xr[j]) * s;
            y[j] = gamma ? t * bf16_to_f32(gamma[j]) : t;
        }
        if (fmt == ORACLE_FMT_NVFP4)
            nvfp4_quantise_row(y, D, q + i * qrow, scales + i * K, rounding, seed, (uint64_t)r);
        else
            mx_quantise_row(y, D, q + i * qrow, scales + i * K, rounding, seed, (uint64_t)r, fmt);
    }
    (void)nthreads;
    return 0;
}

int oracle_mxnorm_fwd(const uint16_t *x, int64_t ld_x, const uint16_t *gamma,
                      int64_t n_rows, const int64_t *row_ids, int64_t D, double p,
                      const float *G_in, uint8_t *q, uint8_t *scales, float *G_out,
                      int rounding, uint64_t seed, int nthreads)
{
    return oracle_mxnorm_fwd_ex(x, ld_x, gamma, n_rows, row_ids, D, p, G_in, q, scales, G_out,
                                rounding, seed, 0, ORACLE_FMT_E4M3, nthreads);
}

/* ------------------------------------------------ MXCast [MX 1.2][RC] */

/* Stand-alone MX quantisation of x (no normalisation): y = x, or, with a gain
   gamma, y = fl32(x_j * gamma_j) -- the folded weight W' of MXNormLinear
   [MX 2.3] when x is a weight stored one output feature per row and gamma
   runs along the input features. */
int oracle_mx_cast_ex(const uint16_t *x, int64_t ld_x, const uint16_t *gamma, int64_t n_rows,
                      const int64_t *row_ids, int64_t D, uint8_t *q, uint8_t *scales,
                      int rounding, uint64_t seed, int fmt, int nthreads)
{
    if (D <= 0 || D % ORACLE_BLOCK != 0) return -1;
    if (fmt != ORACLE_FMT_E4M3 && fmt != ORACLE_FMT_E2M1 && fmt != ORACLE_FMT_NVFP4) return -1;
    int64_t K = D / ((fmt == ORACLE_FMT_NVFP4) ? NVFP4_BLOCK : ORACLE_BLOCK);
    const int64_t qrow = (fmt == ORACLE_FMT_E4M3) ? D : D / 2;
#ifdef _OPENMP
    if (nthreads <= 0) nthreads = omp_get_max_threads();
#pragma omp parallel for schedule(dynamic, 4) num_threads(nthreads)
#endif
    for (int64_t i = 0; i < n_rows; ++i) {
        int64_t r = pick_row(row_ids, i);
        const uint16_t *xr = row_ptr(x, ld_x, r);
        float y[D];
        for (int64_t j = 0; j < D; ++j) {
            float t = bf16_to_f32(xr[j]);
            y[j] = gamma ? t * bf16_to_f32(gamma[j]) : t;
        }
        if (fmt == ORACLE_FMT_NVFP4)
            nvfp4_quantise_row(y, D, q + i * qrow, scales + i * K, rounding, seed, (uint64_t)r);
        else
            mx_quantise_row(y, D, q + i * qrow, scales + i * K, rounding, seed, (uint64_t)r, fmt);
    }
    (void)nthreads;
    return 0;
}

int oracle_mxfp8_cast(const uint16_t *x, int64_t ld_x, int64_t n_rows, const int64_t *row_ids,
                      int64_t D, uint8_t *q, uint8_t *scales, int rounding, uint64_t seed,
                      int nthreads)
{
    return oracle_mx_cast_ex(x, ld_x, NULL, n_rows, row_ids, D, q, scales, rounding, seed,
                             ORACLE_FMT_E4M3, nthreads);
}

/* ------------------------------------------------- RMSNorm [MX 1.2, 2.2] */

/* y = bf16( x / sqrt(mean(x^2) + eps) * gamma ), evaluated in double and
   rounded to bf16 once.  gamma may be NULL (taken as 1). */
int oracle_rmsnorm(const uint16_t *x, int64_t ld_x, const uint16_t *gamma, int64_t n_rows,
                   const int64_t *row_ids, int64_t D, float eps, uint16_t *y, int nthreads)
{
    if (D <= 0) return -1;
#ifdef _OPENMP
    if (nthreads <= 0) nthreads = omp_get_max_threads();
#pragma omp parallel for schedule(dynamic, 4) num_threads(nthreads)
#endif
    for (int64_t i = 0; i < n_rows; ++i) {
        const uint16_t *xr = row_ptr(x, ld_x, pick_row(row_ids, i));
        double ss = 0.0;
        for (int64_t j = 0; j < D; ++j) {
            double v = bf16_to_f32(xr[j]);
            ss += v * v;
        }
        double rinv = 1.0 / sqrt(ss / (double)D + (double)eps);
        for (int64_t j = 0; j < D; ++j) {
            double g = gamma ? (double)bf16_to_f32(gamma[j]) : 1.0;
            y[i * D + j] = bf16_rne_from_double((double)bf16_to_f32(xr[j]) * rinv * g);
        }
    }
    (void)nthreads;
    return 0;
}

/* -------------------------------------------- MXNorm backward [MX 2.3] */

/*
 * Straight-through estimator: the cast is taken as the identity and the
 * normalisation's gradient is the RMSNorm one, with the forward's scale G:
 *   g   = gamma * dy                   (gamma = 1 when NULL)
 *   dx  = ( g - x * (x . g) / (x . x) ) / G
 *   dgamma_j = sum_rows dy_j * x_j / G
 * When true_rms != 0 the variant with the row's true RMS in place of G is
 * computed instead (dx scaled by G/rms).  A row with G = 0 contributes 0.
 * dx is double [n_rows*D]; dgamma is double [D] summed over the selected rows
 * (may be NULL).  Serial: the dgamma sum runs over rows in index order.
 */
int oracle_mxnorm_bwd(const uint16_t *x, const uint16_t *dy, const uint16_t *gamma,
                      const float *G, int64_t n_rows, const int64_t *row_ids, int64_t D,
                      int true_rms, double *dx, double *dgamma)
{
    if (D <= 0) return -1;
    if (dgamma) for (int64_t j = 0; j < D; ++j) dgamma[j] = 0.0;
    for (int64_t i = 0; i < n_rows; ++i) {
        int64_t r = pick_row(row_ids, i);
        const uint16_t *xr = x + r * D, *dyr = dy + r * D;
        double xx = 0.0, xg = 0.0;
        for (int64_t j = 0; j < D; ++j) {
            double xv = bf16_to_f32(xr[j]);
            double g = (gamma ? (double)bf16_to_f32(gamma[j]) : 1.0) * bf16_to_f32(dyr[j]);
            xx += xv * xv;
            xg += xv * g;
        }
        double Gr = (double)G[i];
        if (true_rms) Gr = sqrt(xx / (double)D);
        for (int64_t j = 0; j < D; ++j) {
            double xv = bf16_to_f32(xr[j]);
            double g = (gamma ? (double)bf16_to_f32(gamma[j]) : 1.0) * bf16_to_f32(dyr[j]);
            if (Gr == 0.0 || xx == 0.0) { dx[i * D + j] = 0.0; continue; }
            dx[i * D + j] = (g - xv * xg / xx) / Gr;
            if (dgamma) dgamma[j] += (double)bf16_to_f32(dyr[j]) * xv / (double)G[i];
        }
    }
    return 0;
}

/* ---------------------------------------- block-scaled GEMM [MX 2.3][RC] */

/*
 * C[i][j] = sum_k A(i,k) * B(j,k), each operand dequantised as
 * value(code) * 2^(scale - 127), scales per 32 consecutive k.  A codes [M, K]
 * row-major, A scales [M, K/32]; B codes [N, K] (K contiguous), B scales
 * [N, K/32].  Computes the listed (i, j) entries in double.
 */
static double e4m3_decode_signed(uint8_t c)
{
    double v = oracle_e4m3_value(c & 0x7F);
    if ((c & 0x7F) == 0x7F) v = NAN;
    return (c & 0x80) ? -v : v;
}

int oracle_mxfp8_gemm_entries(const uint8_t *aq, const uint8_t *as, const uint8_t *bq,
                              const uint8_t *bs, int64_t M, int64_t N, int64_t K,
                              int64_t n_entries, const int64_t *ii, const int64_t *jj,
                              double *c, int nthreads)
{
    if (K % ORACLE_BLOCK != 0) return -1;
    int64_t KB = K / ORACLE_BLOCK;
#ifdef _OPENMP
    if (nthreads <= 0) nthreads = omp_get_max_threads();
#pragma omp parallel for schedule(static) num_threads(nthreads)
#endif
    for (int64_t t = 0; t < n_entries; ++t) {
        int64_t i = ii[t], j = jj[t];
        double acc = 0.0;
        if (i < 0 || i >= M || j < 0 || j >= N) { c[t] = NAN; continue; }
        for (int64_t k = 0; k < K; ++k) {
            int ea = (int)as[i * KB + k / ORACLE_BLOCK] - 127;
            int eb = (int)bs[j * KB + k / ORACLE_BLOCK] - 127;
            double a = ldexp(e4m3_decode_signed(aq[i * K + k]), ea);
            double b = ldexp(e4m3_decode_signed(bq[j * K + k]), eb);
            acc += a * b;
        }
        c[t] = acc;
    }
    (void)nthreads;
    return 0;
}

/* --------------------------------------------------------- table helpers */

/* Codes of n fp32 values (RNE or SR with the given words), for the pins. */
void oracle_e4m3_rne_many(const float *v, int64_t n, uint8_t *out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_e4m3_rne(v[i]);
}

void oracle_e4m3_sr_many(const float *v, const uint32_t *r, int64_t n, uint8_t *out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_e4m3_sr(v[i], r[i]);
}

void oracle_e8m0_exponent_many(const float *a, int64_t n, int32_t *out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_e8m0_exponent(fabs((double)a[i]));
}

void oracle_e2m1_rne_many(const float *v, int64_t n, uint8_t *out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_e2m1_rne(v[i]);
}

void oracle_e2m1_sr_many(const float *v, const uint32_t *r, int64_t n, uint8_t *out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_e2m1_sr(v[i], r[i]);
}

void oracle_nvfp4_scale_code_many(const float *a, int64_t n, int32_t *out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_nvfp4_scale_code(fabs((double)a[i]));
}

void oracle_mx_exponent_many(const float *a, int64_t n, double elem_max, int32_t *out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_mx_exponent(fabs((double)a[i]), elem_max);
}

void oracle_sr_words(uint64_t seed, const uint64_t *idx, int64_t n, uint32_t *out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = sr_word(seed, idx[i]);
}

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
