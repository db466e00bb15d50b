/*
 * formats.c -- the three number formats of the method and their exact encoders.
 * TEST INFRASTRUCTURE (see nv4_oracle.h).
 *
 * E2M1  [CAL] format line; values listed in [FP4] 1.1: 1 sign, 2 exponent (bias 1),
 *       1 mantissa bit; magnitudes {0, 0.5, 1, 1.5, 2, 3, 4, 6}.
 * E4M3  [CAL] format line, [FLOW] 3.4 (divisor 448 = largest E4M3 value): "fn" variant,
 *       bias 7, subnormals m*2^-9, 0x7F/0xFF are NaN, no infinity.
 * E8M0  [CAST] section 1/2 and [FP4] 1.2: a pure power of two 2^(code-127), 0xFF is NaN.
 *
 * Encoders round the EXACT real quotient to the nearest representable value, ties
 * to the even code, saturating at the largest finite value.  The decision is an
 * exact comparison of the numerator with midpoint*divisor; exactness of that FP64
 * product is argued at each encoder.
 */
#include "nv4_oracle.h"

#include <math.h>
#include <string.h>

double orc_e2m1_value(unsigned code)
{
    unsigned e = (code >> 1) & 3u, m = code & 1u;
    double mag = (e == 0) ? 0.5 * (double)m : ldexp(1.0 + 0.5 * (double)m, (int)e - 1);
    return (code & 8u) ? -mag : mag;
}

double orc_e4m3_value(unsigned code)
{
    unsigned e = (code >> 3) & 15u, m = code & 7u;
    if ((code & 0x7Fu) == 0x7Fu) return NAN;
    double mag = (e == 0) ? ldexp((double)m, -9) : ldexp(1.0 + (double)m / 8.0, (int)e - 7);
    return (code & 0x80u) ? -mag : mag;
}

double orc_e8m0_value(unsigned code)
{
    if ((code & 0xFFu) == 0xFFu) return NAN;
    return ldexp(1.0, (int)(code & 0xFFu) - 127);
}

/* Index into vals[0..n-1] (strictly increasing, non-negative) of the value nearest to
 * num/den, ties to the even index, saturating at n-1.  Callers guarantee mid*den is
 * exact, so every comparison below is exact. */
static unsigned nearest_index(double num, double den, const double* vals, unsigned n)
{
    for (unsigned k = 0; k + 1 < n; ++k) {
        double mid = 0.5 * (vals[k] + vals[k + 1]);
        double t = mid * den;
        if (num < t) return k;
        if (num == t) return (k & 1u) ? k + 1 : k;
    }
    return n - 1;
}

/* E4M3 block-scale code for the real num/den, num >= 0.
 * Exactness: E4M3 values have at most 4 significant bits, so a midpoint of two
 * neighbours has at most 5; den is 6*s2 with s2 an FP32 value (26 bits) or a power
 * of two; the product has at most 31 significant bits and fits FP64 exactly.
 * den == 0 (a zero per-tensor scale) gives code 0: the block is all zeros. */
static double e4m3_vals[127];

/* Filled once when the library is loaded, before any caller thread exists. */
__attribute__((constructor)) static void init_e4m3_vals(void)
{
    for (unsigned c = 0; c < 127; ++c) e4m3_vals[c] = orc_e4m3_value(c);
}

unsigned orc_e4m3_encode(double num, double den)
{
    if (!(den > 0.0)) return 0u;
    return nearest_index(num, den, e4m3_vals, 127u);
}

/* E2M1 code of x under the effective block scale S: sign bit = signbit(x), magnitude
 * nearest to |x|/S.  Exactness: grid midpoints {0.25 .. 5} have at most 3 significant
 * bits and S is FP32 (24 bits), so mid*S has at most 27 bits.  S == 0 gives magnitude 0. */
unsigned orc_e2m1_encode(double x, double S)
{
    static const double grid[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};
    unsigned sign = signbit(x) ? 8u : 0u;
    if (!(S > 0.0)) return sign;
    return sign | nearest_index(fabs(x), S, grid, 8u);
}

/* Second-level per-tensor scale s2 = amax/6/448 ([FLOW] 3.4), rounded ONCE to FP32.
 * The FP64 quotient followed by the FP32 cast is the correctly rounded single result:
 * double rounding is innocuous for division when 53 >= 2*24+2 (S. A. Figueroa, "When is
 * double rounding innocuous?", ACM SIGNUM Newsletter 30(3), 1995). */
float orc_s2_from_amax(float amax)
{
    return (float)((double)amax / 2688.0);
}

double orc_bf16_value(uint16_t bits)
{
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

/* Round a finite f to the nearest value with p significand bits and minimum normal
 * exponent emin (gradual underflow below it), ties to even; magnitudes that round
 * above maxv overflow to infinity. */
static double round_to_format(double f, int p, int emin, double maxv)
{
    if (f == 0.0 || isnan(f) || isinf(f)) return f;
    int e;
    (void)frexp(f, &e);               /* |f| in [2^(e-1), 2^e) */
    int lead = e - 1;
    if (lead < emin) lead = emin;
    double quantum = ldexp(1.0, lead - (p - 1));
    double r = nearbyint(f / quantum) * quantum; /* division by a power of two is exact */
    if (fabs(r) > maxv) return copysign(INFINITY, f);
    return r;
}

uint16_t orc_f32_to_bf16(float f)
{
    if (isnan(f)) return (uint16_t)(signbit(f) ? 0xFFC0u : 0x7FC0u);
    double r = round_to_format((double)f, 8, -126, ldexp(255.0, 120)); /* max bf16 = (2-2^-7)*2^127 */
    float rf = (float)r;  /* exact: r has 8 significant bits */
    uint32_t u;
    memcpy(&u, &rf, 4);
    return (uint16_t)(u >> 16);
}

uint16_t orc_f32_to_f16(float f)
{
    if (isnan(f)) return (uint16_t)(signbit(f) ? 0xFE00u : 0x7E00u);
    double r = round_to_format((double)f, 11, -14, 65504.0);
    uint16_t sign = signbit(r) ? 0x8000u : 0u;
    double a = fabs(r);
    if (isinf(a)) return (uint16_t)(sign | 0x7C00u);
    if (a == 0.0) return sign;
    if (a < ldexp(1.0, -14)) /* subnormal: a = mant * 2^-24 */
        return (uint16_t)(sign | (uint16_t)(a / ldexp(1.0, -24)));
    int e;
    double fr = frexp(a, &e);         /* a = fr*2^e, fr in [0.5,1) */
    unsigned exp = (unsigned)(e - 1 + 15);
    unsigned mant = (unsigned)((fr * 2.0 - 1.0) * 1024.0);
    return (uint16_t)(sign | (exp << 10) | mant);
}
