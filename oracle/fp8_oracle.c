/*
 * fp8_oracle.c — plain, slow, obviously-correct CPU oracle for the FP8-AMAX
 * scaled linear layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call, link or load
 * this file: only the test-suite, the smoke check and the CPU-baseline /
 * reference leg of the benchmark use it.  It shares no code, header, table or
 * constant with the CUDA library: every number below is written out here from
 * the definitions it cites.
 *
 * Sources (by page title and section):
 *   [P1]  "Training and inference of large language models using 8-bit floating
 *         point" (Perez, Zhang et al., review page), section "Proposed method":
 *         FP8-AMAX takes the per-tensor maximum absolute value of weights,
 *         activations and gradients; compute_bias derives an exponent bias from
 *         log2 of the ratio between the format maximum and that amax, with a
 *         configurable margin; the input is scaled before the FP8 cast and the
 *         matmul output is unscaled afterwards; weights and activations use
 *         FP8_E4, gradients FP8_E5.
 *   [P1-abs] same page, "Abstract": per-tensor scales for weights, gradients and
 *         activations, updated dynamically.
 *   [OCP]  the OCP 8-bit floating point formats E4M3 (no infinities, one NaN
 *         mantissa pattern, largest finite 448) and E5M2 (IEEE-like, largest
 *         finite 57344) — the two formats the page calls FP8_E4 and FP8_E5.
 *
 * Readings taken where the page is silent (each one is listed with its reason
 * in the design notes):
 *   - bias = floor(log2(fmt_max / amax)) - margin  (floor: the largest power of
 *     two that keeps amax * 2^bias <= fmt_max);
 *   - amax == 0, NaN or inf  ->  bias = 0 (log2 undefined / meaningless);
 *   - the cast rounds to nearest, ties to even, and saturates finite overflow to
 *     +-fmt_max ("satfinite"); NaN stays NaN; FP8 subnormals are kept;
 *   - the matmul accumulates the dequantised FP8 products exactly (fp64 here)
 *     and multiplies by 2^-(biasA + biasB) once at the end.
 *
 * Parity pins live in tests/test_oracle_*.py.  Every function here is pinned.
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <string.h>

#define FMT_E4M3 0
#define FMT_E5M2 1

/* ------------------------------------------------------------------------- */
/* FP8 decoding: the format definitions [OCP].                               */
/* ------------------------------------------------------------------------- */

/* Value of an FP8 code, exactly, as a double.  E4M3: 1 sign, 4 exponent bits
 * (bias 7), 3 mantissa bits, S.1111.111 is NaN, no infinity.  E5M2: 1 sign,
 * 5 exponent bits (bias 15), 2 mantissa bits, S.11111.00 is infinity,
 * S.11111.{01,10,11} are NaN.  Exponent field 0 is subnormal: m * 2^(1-bias-mbits). */
double oracle_fp8_decode(uint8_t code, int fmt)
{
    int sign = (code >> 7) & 1;
    int ebits = (fmt == FMT_E4M3) ? 4 : 5;
    int mbits = (fmt == FMT_E4M3) ? 3 : 2;
    int ebias = (fmt == FMT_E4M3) ? 7 : 15;
    int efield = (code >> mbits) & ((1 << ebits) - 1);
    int mfield = code & ((1 << mbits) - 1);
    int emax_field = (1 << ebits) - 1;
    double mag;

    if (fmt == FMT_E4M3 && efield == emax_field && mfield == (1 << mbits) - 1)
        return NAN;
    if (fmt == FMT_E5M2 && efield == emax_field)
        return mfield == 0 ? (sign ? -INFINITY : INFINITY) : NAN;

    if (efield == 0)
        mag = ldexp((double)mfield, 1 - ebias - mbits);
    else
        mag = ldexp((double)((1 << mbits) + mfield), efield - ebias - mbits);
    return sign ? -mag : mag;
}

/* Largest finite value of a format, from its definition: 1.75 * 2^8 = 448 for
 * E4M3 (1.110 x 2^(15-7)), 1.75 * 2^15 = 57344 for E5M2 (1.11 x 2^(30-15)). */
double oracle_fmt_max(int fmt)
{
    return fmt == FMT_E4M3 ? 448.0 : 57344.0;
}

/* Code of the largest finite positive value (0x7E for E4M3, 0x7B for E5M2). */
static uint8_t max_finite_code(int fmt)
{
    return fmt == FMT_E4M3 ? 0x7E : 0x7B;
}

/* ------------------------------------------------------------------------- */
/* FP8 encoding: round to the NEAREST representable value, ties to the code   */
/* whose mantissa LSB is 0 (even), overflow saturates (satfinite).            */
/* Written as a search over the sorted list of the format's non-negative      */
/* finite values, so that "nearest" is literally what is computed.            */
/* ------------------------------------------------------------------------- */

static double g_table[2][128];
static int g_ncodes[2];
static int g_table_ready;

static void build_tables(void)
{
    if (g_table_ready) return;
    for (int fmt = 0; fmt < 2; ++fmt) {
        int n = max_finite_code(fmt) + 1;          /* codes 0x00 .. max, ascending */
        for (int c = 0; c < n; ++c) g_table[fmt][c] = oracle_fp8_decode((uint8_t)c, fmt);
        g_ncodes[fmt] = n;
    }
    g_table_ready = 1;
}

/* Encode v.  saturate != 0: |v| beyond the largest finite value (inf included)
 * gives +-max ("satfinite").  saturate == 0: the IEEE-style overflow rule, used
 * only to check the codec against library conversions: |v| past the midpoint
 * between max and the next binade step (or on it, when the tie's even neighbour
 * is the next step) goes to inf (E5M2) or NaN (E4M3). */
uint8_t oracle_fp8_encode(double v, int fmt, int saturate)
{
    build_tables();
    uint8_t sign = signbit(v) ? 0x80 : 0x00;
    double a = fabs(v);
    const double *t = g_table[fmt];
    int n = g_ncodes[fmt];

    if (isnan(a)) return (uint8_t)(sign | 0x7F);           /* a NaN code in both formats */

    if (a > t[n - 1]) {
        /* Beyond the largest finite value.  The next value the format would
         * have if its exponent went on is max + one max-binade step; the
         * midpoint decides overflow for the non-saturating rule. */
        double step = t[n - 1] - t[n - 2];
        double mid = t[n - 1] + step / 2;
        if (saturate) return (uint8_t)(sign | max_finite_code(fmt));
        /* a tie at mid goes to the neighbour with the even mantissa LSB: the
         * max code itself when it is even (E4M3 0x7E), the next code otherwise
         * (E5M2 0x7B is odd, so the tie goes on to infinity) */
        if (a > mid || (a == mid && (max_finite_code(fmt) & 1)))
            return (uint8_t)(sign | (fmt == FMT_E5M2 ? 0x7C : 0x7F));
        return (uint8_t)(sign | max_finite_code(fmt));
    }

    /* binary search: largest index lo with t[lo] <= a (t[0] == 0 <= a) */
    int lo = 0, hi = n - 1;
    while (lo < hi) {
        int mid = (lo + hi + 1) / 2;
        if (t[mid] <= a) lo = mid; else hi = mid - 1;
    }
    if (t[lo] == a || lo == n - 1) return (uint8_t)(sign | lo);
    double below = a - t[lo], above = t[lo + 1] - a;
    int code;
    if (below < above) code = lo;
    else if (above < below) code = lo + 1;
    else code = (lo % 2 == 0) ? lo : lo + 1;              /* tie: even mantissa LSB */
    return (uint8_t)(sign | code);
}

/* ------------------------------------------------------------------------- */
/* Step 1 — per-tensor amax [P1 "Proposed method", P1-abs].                   */
/* Maximum of |x| over the whole tensor.  NaN propagates (any NaN -> NaN);    */
/* otherwise an inf gives inf.  Result is an fp32 value (every |x| of an fp32 */
/* or bf16 tensor is an fp32 value, so no rounding happens).                  */
/* ------------------------------------------------------------------------- */

static float bf16_to_float(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

float oracle_amax_f32(const float *x, size_t n)
{
    float m = 0.0f;
    int saw_nan = 0;
    for (size_t i = 0; i < n; ++i) {
        float a = fabsf(x[i]);
        if (isnan(a)) saw_nan = 1;
        else if (a > m) m = a;
    }
    return saw_nan ? NAN : m;
}

float oracle_amax_bf16(const uint16_t *x, size_t n)
{
    float m = 0.0f;
    int saw_nan = 0;
    for (size_t i = 0; i < n; ++i) {
        float a = fabsf(bf16_to_float(x[i]));
        if (isnan(a)) saw_nan = 1;
        else if (a > m) m = a;
    }
    return saw_nan ? NAN : m;
}

/* ------------------------------------------------------------------------- */
/* Step 2 — compute_bias [P1 "Proposed method"]: log2 of fmt_max / amax,      */
/* floored, minus the margin.  amax == 0 or non-finite gives 0.               */
/* ------------------------------------------------------------------------- */

int32_t oracle_compute_bias(float amax, int fmt, int margin)
{
    if (!(amax > 0.0f) || isinf(amax)) return 0;             /* 0, NaN, inf */
    double ratio = oracle_fmt_max(fmt) / (double)amax;
    return (int32_t)floor(log2(ratio)) - margin;
}

/* ------------------------------------------------------------------------- */
/* Step 3 — scale, then cast [P1 "Proposed method"]: q = FP8(x * 2^bias).     */
/* x * 2^bias is exact in double for every fp32 x and |bias| < 900.           */
/* ------------------------------------------------------------------------- */

void oracle_cast_scaled_f32(const float *x, size_t n, int32_t bias, int fmt, uint8_t *out)
{
    build_tables();
    #pragma omp parallel for schedule(static)
    for (long long i = 0; i < (long long)n; ++i)
        out[i] = oracle_fp8_encode(ldexp((double)x[i], bias), fmt, 1);
}

void oracle_cast_scaled_bf16(const uint16_t *x, size_t n, int32_t bias, int fmt, uint8_t *out)
{
    build_tables();
    #pragma omp parallel for schedule(static)
    for (long long i = 0; i < (long long)n; ++i)
        out[i] = oracle_fp8_encode(ldexp((double)bf16_to_float(x[i]), bias), fmt, 1);
}

/* Codec over raw fp32 bit patterns, no scaling (for exhaustive checks). */
void oracle_encode_f32_bits(const uint32_t *bits, size_t n, int fmt, int saturate, uint8_t *out)
{
    build_tables();
    #pragma omp parallel for schedule(static)
    for (long long i = 0; i < (long long)n; ++i) {
        float f;
        memcpy(&f, &bits[i], sizeof f);
        out[i] = oracle_fp8_encode((double)f, fmt, saturate);
    }
}

/* ------------------------------------------------------------------------- */
/* Step 4 — FP8 matmuls with the unscale [P1 "Proposed method"]:              */
/*   fwd    Y[t,o]  = sum_i X[t,i]  * W[o,i]   * 2^-(bX + bW)                  */
/*   dgrad  dX[t,i] = sum_o dY[t,o] * W[o,i]   * 2^-(bdY + bW)                 */
/*   wgrad  dW[o,i] = sum_t dY[t,o] * X[t,i]   * 2^-(bdY + bX)                 */
/* All operands are row-major FP8 codes: X [T,in], W [out,in], dY [T,out].    */
/* Each output is the fp64 sum of the exactly dequantised products, then one  */
/* ldexp.  A second output holds the same sum over |products| (the error      */
/* scale used by the tolerance).                                              */
/* ------------------------------------------------------------------------- */

/* One output element: sum_k a[k*sa] * b[k*sb], both decoded. */
static void dot_fp8(const uint8_t *a, int64_t sa, int fa,
                    const uint8_t *b, int64_t sb, int fb,
                    int64_t K, int32_t unscale_exp, double *val, double *absval)
{
    double s = 0.0, sabs = 0.0;
    for (int64_t k = 0; k < K; ++k) {
        double p = oracle_fp8_decode(a[k * sa], fa) * oracle_fp8_decode(b[k * sb], fb);
        s += p;
        sabs += fabs(p);
    }
    *val = ldexp(s, unscale_exp);
    if (absval) *absval = ldexp(sabs, unscale_exp);
}

/* Output entries (rows[e], cols[e]) of one pass; pass 0 = fwd, 1 = dgrad,
 * 2 = wgrad.  (A, fa, bias_a) is X for fwd and dY for dgrad / wgrad;
 * (B, fb, bias_b) is W for fwd / dgrad and X for wgrad. */
void oracle_linear_entries(int pass,
                           const uint8_t *A, int fa, int32_t bias_a,
                           const uint8_t *B, int fb, int32_t bias_b,
                           int64_t T, int64_t in, int64_t out,
                           const int64_t *rows, const int64_t *cols, int64_t count,
                           double *val, double *absval)
{
    build_tables();
    int32_t e = -(bias_a + bias_b);
    #pragma omp parallel for schedule(dynamic, 64)
    for (long long j = 0; j < (long long)count; ++j) {
        int64_t r = rows[j], c = cols[j];
        double *av = absval ? &absval[j] : NULL;
        if (pass == 0)        /* Y[t=r, o=c] = sum_i X[r,i] W[c,i] */
            dot_fp8(A + r * in, 1, fa, B + c * in, 1, fb, in, e, &val[j], av);
        else if (pass == 1)   /* dX[t=r, i=c] = sum_o dY[r,o] W[o,c] */
            dot_fp8(A + r * out, 1, fa, B + c, in, fb, out, e, &val[j], av);
        else                  /* dW[o=r, i=c] = sum_t dY[t,r] X[t,c] */
            dot_fp8(A + r, out, fa, B + c, in, fb, T, e, &val[j], av);
    }
}

/* Whole output of one pass, row-major: fwd [T,out], dgrad [T,in], wgrad [out,in]. */
void oracle_linear_full(int pass,
                        const uint8_t *A, int fa, int32_t bias_a,
                        const uint8_t *B, int fb, int32_t bias_b,
                        int64_t T, int64_t in, int64_t out,
                        double *val, double *absval)
{
    build_tables();
    int64_t R = (pass == 2) ? out : T;
    int64_t C = (pass == 0) ? out : in;
    int32_t e = -(bias_a + bias_b);
    #pragma omp parallel for schedule(dynamic, 1)
    for (long long r = 0; r < (long long)R; ++r) {
        for (int64_t c = 0; c < C; ++c) {
            double *v = &val[r * C + c];
            double *av = absval ? &absval[r * C + c] : NULL;
            if (pass == 0)
                dot_fp8(A + r * in, 1, fa, B + c * in, 1, fb, in, e, v, av);
            else if (pass == 1)
                dot_fp8(A + r * out, 1, fa, B + c, in, fb, out, e, v, av);
            else
                dot_fp8(A + r, out, fa, B + c, in, fb, T, e, v, av);
        }
    }
}

int oracle_num_threads(void)
{
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    return 1;
#endif
}
