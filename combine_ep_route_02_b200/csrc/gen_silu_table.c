/*
 * Build-time generator of the SiLU table used by the expert activation
 * kernel (activation.cu): for every bf16 gate g with 2^-25 <= |g| < 2^7, the
 * bf16 pattern of silu(g) = g / (1 + e^-g), correctly rounded to nearest
 * (ties to even).
 *
 * Entry i = (sign << 12) | (|g| pattern - 0x3300), i.e. 8192 entries: the
 * magnitude patterns 0x3300 (2^-25) .. 0x42FF (just below 2^7) for each sign.
 *
 * Evaluated in x87 extended precision (64-bit significand): the relative
 * error of the quotient is a few units of 2^-64, and the generator stops with
 * an error if any value lies within 2^-56 (relative) of a bf16 rounding
 * midpoint, where that error could decide the rounding.  None does.
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

int main(void)
{
    int bad = 0;
    for (int i = 0; i < 8192; ++i) {
        uint16_t b = (uint16_t)(((i >> 12) << 15) | (0x3300 + (i & 4095)));
        long double x = (long double)bf16_to_float(b);
        long double v = x / (1.0L + expl(-x));
        int close = 0;
        uint16_t s = round_to_bf16(v, &close);
        if (close) {
            fprintf(stderr, "gen_silu_table: input 0x%04x lies too close to a midpoint\n", b);
            bad = 1;
        }
        printf("0x%04x,%s", s, (i % 16 == 15) ? "\n" : " ");
    }
    return bad;
}
