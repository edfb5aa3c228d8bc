/*
 * Build-time generator of the SiLU table used by the expert activation
 * kernel (activation.cu): for every one of the 65,536 bf16 gate patterns g,
 * the bf16 pattern of silu(g) = g / (1 + e^-g), correctly rounded to nearest
 * (ties to even).  Entry i is the result for the gate whose bit pattern is i.
 *
 * For 2^-25 <= |g| < 2^7 the value is evaluated in x87 extended precision
 * (64-bit significand): the relative error of the quotient is a few units of
 * 2^-64, and the generator stops with an error if any value lies within
 * 2^-56 (relative) of a bf16 rounding midpoint, where that error could decide
 * the rounding.  None does.  Outside that range the result has closed forms:
 *   |g| < 2^-25: silu(g) - g/2 = g tanh(g/2) / 2 is positive (g and
 *     tanh(g/2) share a sign) and below half a bf16 step of g/2, so the
 *     result is g/2 (exact in fp32) rounded to bf16 with ties toward +inf (a
 *     tie occurs only below 2^-126);
 *   |g| >= 2^7 and +-inf: g for g > 0 and -0 for g < 0 (|g e^g| < 2^-180);
 *   NaN: the gate pattern itself.
 *
 * Usage: gen_silu_table > silu_table.inc  (comma-separated hex values)
 */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>

static float bf16_to_float(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* bf16 pattern of the finite nonzero value v, to nearest (ties to even);
 * sets *close when v is within 2^-56 relative of a midpoint. */
static uint16_t round_to_bf16(long double v, int *close)
{
    uint16_t sign = v < 0 ? 0x8000u : 0u;
    long double a = fabsl(v);
    int e;
    frexpl(a, &e);                    /* 2^(e-1) <= a < 2^e */
    int q_exp = (e - 1 < -126 ? -126 : e - 1) - 7;   /* bf16 step: 8 bits, subnormal below 2^-126 */
    long double n = ldexpl(a, -q_exp);  /* exact: a power-of-two scaling */
    long double fl = floorl(n);
    long double frac = n - fl;
    *close = fabsl(frac - 0.5L) <= ldexpl(n, -56);
    long double r = fl;
    if (frac > 0.5L || (frac == 0.5L && fmodl(fl, 2.0L) != 0.0L)) r = fl + 1.0L;
    long double res = ldexpl(r, q_exp);
    float f = (float)res;             /* a bf16 value: exact in fp32 */
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    if (res >= 0x1p128L) u = 0x7F800000u;
    return (uint16_t)(sign | (u >> 16));
}

/* g/2 rounded to bf16, ties toward +inf: the low 16 bits of the fp32
 * pattern decide, a tie (exactly 0x8000) going up in magnitude for g > 0 and
 * down in magnitude for g < 0. */
static uint16_t half_toward_plus_inf(uint16_t b)
{
    float h = bf16_to_float(b) * 0.5f;
    uint32_t u;
    memcpy(&u, &h, sizeof u);
    return (uint16_t)((u + ((u >> 31) ? 0x7FFFu : 0x8000u)) >> 16);
}

int main(void)
{
    int bad = 0;
    for (int i = 0; i < 65536; ++i) {
        const uint16_t b = (uint16_t)i, a = b & 0x7FFFu;
        uint16_t s;
        if (a > 0x7F80u) {
            s = b;
        } else if (a >= 0x4300u) {
            s = (b & 0x8000u) ? 0x8000u : b;
        } else if (a < 0x3300u) {
            s = half_toward_plus_inf(b);
        } else {
            long double x = (long double)bf16_to_float(b);
            long double v = x / (1.0L + expl(-x));
            int close = 0;
            s = round_to_bf16(v, &close);
            if (close) {
                fprintf(stderr, "gen_silu_table: input 0x%04x lies too close to a midpoint\n", b);
                bad = 1;
            }
        }
        printf("0x%04x,%s", s, (i % 16 == 15) ? "\n" : " ");
    }
    return bad;
}
