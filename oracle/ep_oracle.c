/*
 * ep_oracle.c -- plain, slow, single-threaded CPU restatement of the MoE
 * expert-parallel routing / dispatch-layout / dispatch / combine path.
 *
 * TEST INFRASTRUCTURE.  Only the test suite, the package smoke check and the
 * benchmark's CPU-baseline leg load this code.  It shares no source, header,
 * table or helper with the CUDA library; each side is written from the
 * definitions below.
 *
 * Build: gcc -O2 -std=c11 -ffp-contract=off -fno-fast-math -fPIC -shared -lm
 * (no FMA contraction: every float operation below rounds once, to nearest).
 *
 * Sources of the definitions (page title, then section):
 *  - "Lower latency and higher throughput with multi-node DeepSeek
 *    deployment" (Perplexity blog), section "Expert Parallelism": 256 routed
 *    experts, each token goes to 8 of them and the results are summed with
 *    weights; dispatch and combine are the two all-to-alls around the
 *    experts.  Section "MoE Router": Mixtral routing is the special case of
 *    DeepSeek group routing where the top-K group is all experts.  Section
 *    "Quantization": one activation scale per 128-element vector, M x
 *    ceil_div(K,128) of them, from the maximum absolute value of each
 *    128-element sub-block.
 *  - DeepSeek Open Infra day-4 summary (DualPipe / EPLB / profile data),
 *    section EPLB: group-limited expert routing keeps a token's experts on
 *    as few nodes (groups) as possible.
 *  - DeepEP V2 summary (news.hada.io), sections "Performance" and "Usage for
 *    training, prefill and decoding": FP8 dispatch with BF16 combine; the
 *    dispatch handle carries per-expert receive counts for the GEMM.
 *  - The method as specified for this library fixes what the pages leave
 *    open: sigmoid gating with a selection bias, group score = sum of the
 *    top-2 scores of a group, ties to the lower index, scale = amax/448 with
 *    round-to-nearest-even into e4m3, rank-major expert-contiguous receive
 *    rows, BF16 combine with fp32 accumulation.
 *
 * Readings where the pages are silent:
 *  R1 sigmoid: s = the exact 1 / (1 + e^-x) rounded once to fp32 (nearest,
 *     ties to even; a tie cannot occur: the value is irrational for x != 0).
 *     It is evaluated in fp64 (error a few units of 2^-53); an element whose
 *     fp64 value lies within 2^-47 (relative) of an fp32 rounding midpoint is
 *     flagged "hard" and decided again in quad precision (113-bit
 *     significand), far closer than any fp32 input comes to a midpoint.
 *  R2 the bias enters selection only: key = fp32_RN(s + b); weights use s.
 *  R3 group score = fp32_RN(k1 + k2), k1 >= k2 the two largest keys.
 *  R4 order: (key desc, index asc) for experts; (score desc, id asc) for
 *     groups.  Output order of top-k = selection order.
 *  R5 weights: w_j = s_j; if renorm: sum = fp32 sum in j order, and when
 *     sum != 0, w_j = fp32_RN(w_j / sum); then w_j = fp32_RN(w_j * scale).
 *  R6 receive rows: sorted by physical expert, then by (token, j); no padding.
 *  R7 e4m3 "fn" (bias 7, max 448, no inf), round to nearest even, saturating
 *     to +-448; q = e4m3(fp32_RN(x / scale)); a block with amax == 0 has
 *     scale 0 and all payload bytes 0x00.
 *  R8 combine: acc = 0; acc = fp32_RN(acc + fp32_RN(w_j * y_j)) in j order;
 *     out = bf16_RNE(acc).
 *  R9 expert activation (SiLU, Perplexity blog section "Quantization"): the
 *     first grouped GEMM's row holds [gate | up], I bf16 each (DeepSeek-V3's
 *     gated SiLU expert).  s = bf16_RN(silu(g)), silu(g) = g / (1 + e^-g),
 *     correctly rounded (fp64 evaluation; silu(-inf) = -0, silu(+inf) =
 *     +inf); h = bf16_RN(fp32_RN(s * u)), as a BF16 model multiplies; then
 *     h is quantised per 128 elements as in R7.
 *  R10 GEMM layout: with a row tile A > 1, expert p's rows start at a
 *     multiple of A and are followed by round_up(cnt, A) - cnt padding rows
 *     (src = -1); expert_off / rank_off / rows_rank count padded rows.
 *  R11 the activation reads the per-expert counts: it processes exactly the
 *     rows [expert_off[p], expert_off[p] + cnt_expert[p]) and leaves padding
 *     and unused rows untouched.
 */
#include <math.h>
#include <quadmath.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_BAD_EXPERT 1
#define ORC_BAD_REPLICA 2

/* ------------------------------------------------------------------ */
/* number formats                                                      */
/* ------------------------------------------------------------------ */

static float bits_to_float(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }
static uint32_t float_to_bits(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }

/* bf16 -> fp32 is exact: the bf16 pattern is the top half of the fp32 one. */
float orc_bf16_decode(uint16_t b) { return bits_to_float((uint32_t)b << 16); }

/* fp32 -> bf16, round to nearest, ties to even (keep 16 high bits). */
uint16_t orc_bf16_encode(float v)
{
    uint32_t u = float_to_bits(v);
    if (isnan(v)) return (uint16_t)((u >> 16) | 0x0040u); /* stay a NaN */
    uint32_t hi = u >> 16, lo = u & 0xFFFFu;
    if (lo > 0x8000u || (lo == 0x8000u && (hi & 1u))) hi += 1u; /* may carry into inf */
    return (uint16_t)hi;
}

/* Round a non-negative double holding an exact value to the nearest
 * integer, ties to even (written out rather than relying on a mode). */
static double round_half_even(double v)
{
    double f = floor(v), d = v - f;
    if (d > 0.5) return f + 1.0;
    if (d < 0.5) return f;
    return (fmod(f, 2.0) == 0.0) ? f : f + 1.0;
}

/* e4m3 "fn": sign | 4-bit exponent (bias 7) | 3-bit mantissa.
 * normal:    (-1)^s 2^(E-7) (1 + m/8),  E = 1..15 (E=15,m=7 is NaN)
 * subnormal: (-1)^s 2^-6 (m/8) = m 2^-9,  E = 0.
 * Largest finite value 448 (0x7E).  Saturating: |v| >= 448 -> 448. */
uint8_t orc_e4m3_encode(float v)
{
    if (isnan(v)) return 0x7F;
    uint8_t sign = (float_to_bits(v) >> 31) ? 0x80 : 0x00;
    double a = fabs((double)v);
    if (a >= 448.0) return sign | 0x7E;
    if (a < 0.015625) { /* below 2^-6: subnormal grid of step 2^-9 */
        double m = round_half_even(a * 512.0); /* 0..8, 8 is the smallest normal */
        return sign | (uint8_t)m;
    }
    int e;
    double fr = frexp(a, &e);    /* a = fr * 2^e, fr in [0.5, 1) */
    int E = e - 1;               /* a = (2 fr) 2^E, 2 fr in [1, 2) */
    double m = round_half_even((2.0 * fr - 1.0) * 8.0);
    if (m == 8.0) { m = 0.0; E += 1; }
    /* a < 448 keeps the result at or below 448 = 2^8 * 1.75 */
    return sign | (uint8_t)(((E + 7) << 3) | (int)m);
}

float orc_e4m3_decode(uint8_t c)
{
    int s = c >> 7, E = (c >> 3) & 0xF, m = c & 7;
    double v;
    if (E == 15 && m == 7) return NAN;
    if (E == 0) v = ldexp((double)m, -9);
    else v = ldexp(1.0 + m / 8.0, E - 7);
    return (float)(s ? -v : v);
}

/* ------------------------------------------------------------------ */
/* routing                                                             */
/* ------------------------------------------------------------------ */

/* fp64 sigmoid and whether it lies within 2^-47 (relative) of an fp32
 * rounding midpoint (then fp64 cannot be trusted to round it). */
static double sigmoid_fp64(float x, int *hard)
{
    double v = 1.0 / (1.0 + exp(-(double)x));
    float f = (float)v;
    double fd = (double)f;
    float other = (v >= fd) ? nextafterf(f, INFINITY) : nextafterf(f, -INFINITY);
    double mid = 0.5 * (fd + (double)other); /* exact: adjacent floats */
    *hard = fabs(v - mid) <= ldexp(fabs(v), -47);
    return v;
}

/* R1: the sigmoid correctly rounded to fp32, with the hard-case flag. */
float orc_sigmoid(float x, int *hard)
{
    int h = 0;
    double v = sigmoid_fp64(x, &h);
    if (hard) *hard = h;
    float f = (float)v;
    if (!h) return f;
    /* near a midpoint: the two fp32 neighbours, and the side of their
     * midpoint on which the quad-precision value lies */
    double fd = (double)f;
    float other = (v >= fd) ? nextafterf(f, INFINITY) : nextafterf(f, -INFINITY);
    float lo = fd < (double)other ? f : other;
    float hi = fd < (double)other ? other : f;
    __float128 q = 1.0Q / (1.0Q + expq(-(__float128)x));
    __float128 m = ((__float128)lo + (__float128)hi) / 2; /* exact */
    if (q > m) return hi;
    if (q < m) return lo;
    return (float_to_bits(lo) & 1u) ? hi : lo; /* a tie: to even (never met) */
}

/* Bit patterns b in [first, first + count) whose fp32 value's sigmoid is
 * hard (see sigmoid_fp64); NaN patterns are skipped.  Writes up to cap of
 * them to out and returns how many there are. */
uint32_t orc_sigmoid_hard_scan(uint32_t first, uint32_t count, uint32_t *out, uint32_t cap)
{
    uint32_t n = 0;
    for (uint32_t i = 0; i < count; ++i) {
        uint32_t b = first + i;
        float x = bits_to_float(b);
        if (isnan(x)) continue;
        int h = 0;
        sigmoid_fp64(x, &h);
        if (h) {
            if (n < cap) out[n] = b;
            ++n;
        }
    }
    return n;
}

/*
 * Sigmoid-gated, group-limited top-k routing, one token at a time.
 * logits [T,E], bias [E] or NULL (all zero), outputs topk_idx [T,k],
 * topk_w [T,k]; hard_tok [T] (optional) marks tokens holding a hard sigmoid.
 * Groups are n_group runs of E/n_group consecutive experts.
 * Returns 0, or -1 (writing nothing) for a configuration the method does
 * not define: E not a multiple of n_group, topk_group outside [1, n_group],
 * k outside [1, (E/n_group) * topk_group], or, with more than one group,
 * groups of a single expert (R3 scores a group by its TWO largest keys).
 */
int orc_route(const float *logits, const float *bias, int T, int E,
              int n_group, int topk_group, int k, float routed_scale,
              int renorm, int32_t *topk_idx, float *topk_w, uint8_t *hard_tok)
{
    if (T < 0 || E < 1 || n_group < 1 || E % n_group != 0) return -1;
    if (topk_group < 1 || topk_group > n_group) return -1;
    if (k < 1 || k > (E / n_group) * topk_group) return -1;
    if (n_group > 1 && E / n_group < 2) return -1;

    float *s = malloc(sizeof(float) * (size_t)E);
    float *key = malloc(sizeof(float) * (size_t)E);
    float *gscore = malloc(sizeof(float) * (size_t)n_group);
    unsigned char *allowed = malloc((size_t)E);
    unsigned char *taken = malloc((size_t)E);
    unsigned char *gsel = malloc((size_t)n_group);
    int gs = E / n_group;

    for (int t = 0; t < T; ++t) {
        const float *row = logits + (size_t)t * E;
        int hard_any = 0;
        for (int e = 0; e < E; ++e) {
            int h = 0;
            s[e] = orc_sigmoid(row[e], &h);
            hard_any |= h;
            key[e] = s[e] + (bias ? bias[e] : 0.0f); /* R2 */
        }

        if (n_group > 1) {
            /* R3: score of a group = sum of its two largest keys */
            for (int g = 0; g < n_group; ++g) {
                int i1 = g * gs;
                for (int e = g * gs + 1; e < (g + 1) * gs; ++e)
                    if (key[e] > key[i1]) i1 = e;
                int i2 = -1;
                for (int e = g * gs; e < (g + 1) * gs; ++e) {
                    if (e == i1) continue;
                    if (i2 < 0 || key[e] > key[i2]) i2 = e;
                }
                gscore[g] = key[i1] + key[i2];
            }
            /* keep the topk_group best groups, ties to the lower group id */
            memset(gsel, 0, (size_t)n_group);
            for (int r = 0; r < topk_group; ++r) {
                int best = -1;
                for (int g = 0; g < n_group; ++g)
                    if (!gsel[g] && (best < 0 || gscore[g] > gscore[best])) best = g;
                gsel[best] = 1;
            }
            for (int e = 0; e < E; ++e) allowed[e] = gsel[e / gs];
        } else {
            memset(allowed, 1, (size_t)E);
        }

        /* top-k among allowed experts by (key desc, index asc) */
        memset(taken, 0, (size_t)E);
        int32_t *idx = topk_idx + (size_t)t * k;
        float *w = topk_w + (size_t)t * k;
        for (int j = 0; j < k; ++j) {
            int best = -1;
            for (int e = 0; e < E; ++e)
                if (allowed[e] && !taken[e] && (best < 0 || key[e] > key[best])) best = e;
            taken[best] = 1;
            idx[j] = best;
            w[j] = s[best];
        }
        /* R5 */
        if (renorm) {
            float sum = 0.0f;
            for (int j = 0; j < k; ++j) sum = sum + w[j];
            if (sum != 0.0f)
                for (int j = 0; j < k; ++j) w[j] = w[j] / sum;
        }
        for (int j = 0; j < k; ++j) w[j] = w[j] * routed_scale;
        if (hard_tok) hard_tok[t] = (uint8_t)hard_any;
    }
    free(s); free(key); free(gscore); free(allowed); free(taken); free(gsel);
    return 0;
}

/* ------------------------------------------------------------------ */
/* dispatch layout                                                     */
/* ------------------------------------------------------------------ */

int orc_layout_aligned(const int32_t *topk_idx, int T, int k, int E, int P, int R,
                       const int32_t *phys_of, const int32_t *n_rep, int max_rep,
                       int row_align, int32_t *cnt_expert, int32_t *expert_off,
                       int32_t *rows_rank, int32_t *rank_off, int32_t *tok_rank,
                       uint8_t *in_rank, int32_t *slot, int32_t *src);

/* physical expert of pair (t, j); -1 (and a status bit) when invalid */
static int phys_expert(const int32_t *topk_idx, int t, int j, int k, int E, int P,
                       const int32_t *phys_of, const int32_t *n_rep, int max_rep,
                       int *status)
{
    int e = topk_idx[(size_t)t * k + j];
    if (e < 0 || e >= E) { *status |= ORC_BAD_EXPERT; return -1; }
    if (!phys_of) return e;
    int n = n_rep[e];
    if (n < 1 || n > max_rep) { *status |= ORC_BAD_REPLICA; return -1; }
    int p = phys_of[(size_t)e * max_rep + (t % n)];
    if (p < 0 || p >= P) { *status |= ORC_BAD_REPLICA; return -1; }
    return p;
}

/*
 * Per-expert / per-rank counts, prefix sums, and slots (R6).
 * Physical expert p lives on rank p / (P/R).  Returns the status bits.
 * Arrays: cnt_expert[P], expert_off[P+1], rows_rank[R], rank_off[R+1],
 * tok_rank[R], in_rank[T*R], slot[T*k], src[T*k].
 */
int orc_layout(const int32_t *topk_idx, int T, int k, int E, int P, int R,
               const int32_t *phys_of, const int32_t *n_rep, int max_rep,
               int32_t *cnt_expert, int32_t *expert_off, int32_t *rows_rank,
               int32_t *rank_off, int32_t *tok_rank, uint8_t *in_rank,
               int32_t *slot, int32_t *src)
{
    return orc_layout_aligned(topk_idx, T, k, E, P, R, phys_of, n_rep, max_rep, 1,
                              cnt_expert, expert_off, rows_rank, rank_off, tok_rank,
                              in_rank, slot, src);
}

/*
 * The same layout with every expert's first receive row a multiple of
 * row_align (the row tile of a grouped GEMM consuming the receive buffer,
 * the "GEMM layout" of the DeepEP V2 summary): expert p occupies rows
 * [expert_off[p], expert_off[p] + cnt_expert[p]) followed by
 * round_up(cnt, row_align) - cnt padding rows whose src is -1.
 * expert_off, rows_rank and rank_off count padded rows; cnt_expert and
 * tok_rank do not.  src has expert_off[P] entries.
 */
int orc_layout_aligned(const int32_t *topk_idx, int T, int k, int E, int P, int R,
                       const int32_t *phys_of, const int32_t *n_rep, int max_rep,
                       int row_align, int32_t *cnt_expert, int32_t *expert_off,
                       int32_t *rows_rank, int32_t *rank_off, int32_t *tok_rank,
                       uint8_t *in_rank, int32_t *slot, int32_t *src)
{
    int status = 0;
    int epr = P / R;
    int32_t *fill = calloc((size_t)P, sizeof(int32_t));

    for (int p = 0; p < P; ++p) cnt_expert[p] = 0;
    for (int t = 0; t < T; ++t)
        for (int j = 0; j < k; ++j) {
            int p = phys_expert(topk_idx, t, j, k, E, P, phys_of, n_rep, max_rep, &status);
            if (p >= 0) cnt_expert[p] += 1;
        }

    expert_off[0] = 0;
    for (int p = 0; p < P; ++p) {
        int padded = (cnt_expert[p] + row_align - 1) / row_align * row_align;
        expert_off[p + 1] = expert_off[p] + padded;
    }
    for (int p = 0; p < P; ++p)
        for (int r = expert_off[p] + cnt_expert[p]; r < expert_off[p + 1]; ++r) src[r] = -1;

    for (int t = 0; t < T; ++t)
        for (int j = 0; j < k; ++j) {
            int dummy = 0;
            int p = phys_expert(topk_idx, t, j, k, E, P, phys_of, n_rep, max_rep, &dummy);
            if (p < 0) { slot[(size_t)t * k + j] = -1; continue; }
            int sl = expert_off[p] + fill[p];
            fill[p] += 1;
            slot[(size_t)t * k + j] = sl;
            src[sl] = t * k + j;
        }

    for (int r = 0; r < R; ++r) {
        rank_off[r] = expert_off[r * epr];
        rows_rank[r] = expert_off[(r + 1) * epr] - expert_off[r * epr];
    }
    rank_off[R] = expert_off[P];

    memset(in_rank, 0, (size_t)T * R);
    for (int t = 0; t < T; ++t)
        for (int j = 0; j < k; ++j) {
            int dummy = 0;
            int p = phys_expert(topk_idx, t, j, k, E, P, phys_of, n_rep, max_rep, &dummy);
            if (p >= 0) in_rank[(size_t)t * R + p / epr] = 1;
        }
    for (int r = 0; r < R; ++r) {
        int c = 0;
        for (int t = 0; t < T; ++t) c += in_rank[(size_t)t * R + r];
        tok_rank[r] = c;
    }
    free(fill);
    return status;
}

/* ------------------------------------------------------------------ */
/* dispatch: permute (+ 1x128 FP8 quantise)                            */
/* ------------------------------------------------------------------ */

/* Quantise one bf16 row of H (H % 128 == 0) into e4m3 codes and H/128
 * fp32 scales (R7). */
void orc_quantize_row(const uint16_t *x, int H, uint8_t *q, float *scales)
{
    for (int b = 0; b < H / 128; ++b) {
        float amax = 0.0f;
        for (int i = 0; i < 128; ++i) {
            float a = fabsf(orc_bf16_decode(x[b * 128 + i]));
            if (a > amax) amax = a;
        }
        float scale = amax / 448.0f;
        scales[b] = scale;
        for (int i = 0; i < 128; ++i) {
            if (amax == 0.0f) { q[b * 128 + i] = 0x00; continue; }
            float v = orc_bf16_decode(x[b * 128 + i]);
            q[b * 128 + i] = orc_e4m3_encode(v / scale);
        }
    }
}

/*
 * For every token t and j < k, write row x[t] (quantised when fp8) into
 * receive row slot[t,j].  Slots outside [0, n_rows) are skipped.
 * fp8: recv_x is uint8 [n_rows, H], recv_scale fp32 [n_rows, H/128];
 * bf16: recv_x is uint16 [n_rows, H] (bitwise copies), recv_scale unused.
 */
void orc_dispatch(const uint16_t *x, int T, int H, int k, const int32_t *slot,
                  int n_rows, int fp8, void *recv_x, float *recv_scale)
{
    int S = H / 128;
    uint8_t *q = malloc((size_t)H);
    float *sc = malloc(sizeof(float) * (size_t)(S > 0 ? S : 1));
    for (int t = 0; t < T; ++t) {
        const uint16_t *row = x + (size_t)t * H;
        if (fp8) orc_quantize_row(row, H, q, sc);
        for (int j = 0; j < k; ++j) {
            int s = slot[(size_t)t * k + j];
            if (s < 0 || s >= n_rows) continue;
            if (fp8) {
                memcpy((uint8_t *)recv_x + (size_t)s * H, q, (size_t)H);
                memcpy(recv_scale + (size_t)s * S, sc, sizeof(float) * (size_t)S);
            } else {
                memcpy((uint16_t *)recv_x + (size_t)s * H, row, sizeof(uint16_t) * (size_t)H);
            }
        }
    }
    free(q); free(sc);
}

/* ------------------------------------------------------------------ */
/* combine                                                             */
/* ------------------------------------------------------------------ */

/*
 * out[t] = bf16( sum_j w[t,j] * y[slot[t,j]] ), fp32 accumulation in j order
 * (R8).  y bf16 [n_rows, H]; slots outside [0, n_rows) contribute nothing.
 */
void orc_combine(const uint16_t *y, int n_rows, const int32_t *slot, const float *w,
                 int T, int H, int k, uint16_t *out)
{
    float *acc = malloc(sizeof(float) * (size_t)(H > 0 ? H : 1));
    for (int t = 0; t < T; ++t) {
        for (int h = 0; h < H; ++h) acc[h] = 0.0f;
        for (int j = 0; j < k; ++j) {
            int s = slot[(size_t)t * k + j];
            if (s < 0 || s >= n_rows) continue;
            float wj = w[(size_t)t * k + j];
            const uint16_t *yr = y + (size_t)s * H;
            for (int h = 0; h < H; ++h) {
                float prod = wj * orc_bf16_decode(yr[h]);
                acc[h] = acc[h] + prod;
            }
        }
        for (int h = 0; h < H; ++h) out[(size_t)t * H + h] = orc_bf16_encode(acc[h]);
    }
    free(acc);
}

/* ------------------------------------------------------------------ */
/* array forms of the encoders (for exhaustive format checks)          */
/* ------------------------------------------------------------------ */

void orc_e4m3_encode_array(const float *v, size_t n, uint8_t *out)
{
    for (size_t i = 0; i < n; ++i) out[i] = orc_e4m3_encode(v[i]);
}

void orc_bf16_encode_array(const float *v, size_t n, uint16_t *out)
{
    for (size_t i = 0; i < n; ++i) out[i] = orc_bf16_encode(v[i]);
}

void orc_sigmoid_array(const float *x, size_t n, float *out, uint8_t *hard)
{
    for (size_t i = 0; i < n; ++i) {
        int h = 0;
        out[i] = orc_sigmoid(x[i], &h);
        hard[i] = (uint8_t)h;
    }
}

/* ------------------------------------------------------------------ */
/* backward (training): dispatch-backward and combine-backward        */
/* ------------------------------------------------------------------ */
/*
 * DeepEP V2 summary, section "Usage for training, prefill and decoding":
 * the backward of dispatch is a combine and the backward of combine is a
 * dispatch.  Reading: the forward FP8 quantisation is treated as the
 * identity (straight-through), so gradients travel in BF16.
 *
 * dispatch-backward: grad_x[t] = bf16( sum_j grad_recv[slot[t,j]] ), fp32
 * accumulation in j order (the combine of R8 with unit weights).
 */
void orc_dispatch_backward(const uint16_t *grad_recv, int n_rows, const int32_t *slot,
                           int T, int H, int k, uint16_t *grad_x)
{
    float *acc = malloc(sizeof(float) * (size_t)(H > 0 ? H : 1));
    for (int t = 0; t < T; ++t) {
        for (int h = 0; h < H; ++h) acc[h] = 0.0f;
        for (int j = 0; j < k; ++j) {
            int s = slot[(size_t)t * k + j];
            if (s < 0 || s >= n_rows) continue;
            const uint16_t *g = grad_recv + (size_t)s * H;
            for (int h = 0; h < H; ++h) acc[h] = acc[h] + orc_bf16_decode(g[h]);
        }
        for (int h = 0; h < H; ++h) grad_x[(size_t)t * H + h] = orc_bf16_encode(acc[h]);
    }
    free(acc);
}

/*
 * combine-backward, for out[t] = sum_j w[t,j] * y[slot[t,j]]:
 *   grad_y[slot[t,j]] = bf16( fp32(w[t,j] * grad_out[t]) )   (rows of
 *                        invalid slots are not written)
 *   grad_w[t,j]       = sum_h grad_out[t,h] * y[slot[t,j],h], evaluated in
 *                        fp64 and rounded once to fp32 (0 for invalid slots)
 */
void orc_combine_backward(const uint16_t *grad_out, const uint16_t *y, int n_rows,
                          const int32_t *slot, const float *w, int T, int H, int k,
                          uint16_t *grad_y, float *grad_w)
{
    for (int t = 0; t < T; ++t) {
        const uint16_t *g = grad_out + (size_t)t * H;
        for (int j = 0; j < k; ++j) {
            int s = slot[(size_t)t * k + j];
            if (s < 0 || s >= n_rows) { grad_w[(size_t)t * k + j] = 0.0f; continue; }
            float wj = w[(size_t)t * k + j];
            const uint16_t *yr = y + (size_t)s * H;
            double dot = 0.0;
            for (int h = 0; h < H; ++h) {
                float gh = orc_bf16_decode(g[h]);
                grad_y[(size_t)s * H + h] = orc_bf16_encode(wj * gh);
                dot += (double)gh * (double)orc_bf16_decode(yr[h]);
            }
            grad_w[(size_t)t * k + j] = (float)dot;
        }
    }
}

/* ------------------------------------------------------------------ */
/* expert activation: SiLU(gate) * up, then 1x128 FP8 (R9, R11)        */
/* ------------------------------------------------------------------ */

/* Round a finite double to bf16, to nearest, and flag values within 2^-44
 * (relative) of a rounding midpoint.  bf16 keeps 8 significant bits down to
 * 2^-126 and a fixed step of 2^-133 below.  An exact tie goes to the even
 * neighbour, or, with tie_up set, to the neighbour toward +inf (for a value
 * known to lie a hair above v). */
static uint16_t bf16_round_double(double v, int *hard, int tie_up)
{
    uint16_t sign = signbit(v) ? 0x8000u : 0x0000u;
    double a = fabs(v);
    if (hard) *hard = 0;
    if (a == 0.0) return sign;
    double q;
    if (a < 0x1p-126) {
        q = 0x1p-133;
    } else {
        int e;
        frexp(a, &e);            /* 2^(e-1) <= a < 2^e */
        q = ldexp(1.0, e - 1 - 7);
    }
    double n = a / q;            /* exact: a power-of-two scaling */
    double r = round_half_even(n);
    if (tie_up && n - floor(n) == 0.5) r = sign ? floor(n) : floor(n) + 1.0;
    if (hard && !tie_up) *hard = fabs(n - floor(n) - 0.5) <= ldexp(n, -44);
    double res = r * q;
    if (res >= 0x1p128) return sign | 0x7F80u; /* rounds past the largest finite */
    return sign | (uint16_t)(float_to_bits((float)res) >> 16); /* res is a bf16 value */
}

/* R9: SiLU of a bf16 value, correctly rounded to bf16. */
uint16_t orc_silu_bf16(uint16_t g, int *hard)
{
    float gf = orc_bf16_decode(g);
    if (hard) *hard = 0;
    if (isnan(gf)) return (uint16_t)(g | 0x0040u);
    if (isinf(gf)) return gf > 0 ? 0x7F80u : 0x8000u;
    double x = (double)gf;
    /* silu(x) - x/2 = x tanh(x/2) / 2 > 0 for x != 0.  For tiny x that
     * difference is far below fp64 resolution, the fp64 quotient is x/2
     * exactly, and x/2 can be a bf16 midpoint (odd multiples of 2^-134): the
     * exact value lies just above it, so such a tie rounds toward +inf. */
    if (fabs(x) < 0x1p-100) return bf16_round_double(x / 2.0, hard, 1);
    return bf16_round_double(x / (1.0 + exp(-x)), hard, 0);
}

void orc_silu_bf16_array(const uint16_t *g, size_t n, uint16_t *out, uint8_t *hard)
{
    for (size_t i = 0; i < n; ++i) {
        int h = 0;
        out[i] = orc_silu_bf16(g[i], &h);
        hard[i] = (uint8_t)h;
    }
}

/* R9: h[i] = bf16(fp32(silu_bf16(gate[i]) * up[i])) for one row. */
void orc_silu_mul_row(const uint16_t *gate_up, int I, uint16_t *h)
{
    for (int i = 0; i < I; ++i) {
        float s = orc_bf16_decode(orc_silu_bf16(gate_up[i], NULL));
        float u = orc_bf16_decode(gate_up[I + i]);
        float prod = s * u;
        h[i] = orc_bf16_encode(prod);
    }
}

/*
 * Expert activation over the receive rows (R9, R11).  gate_up bf16
 * [n_rows, 2I]; expert_off / cnt_expert select the rows (NULL: every row).
 * fp8: act is e4m3 [n_rows, I] and act_scale fp32 [n_rows, I/128];
 * otherwise act is bf16 [n_rows, I] (h itself).  Rows outside the selection
 * are not written.
 */
void orc_silu_mul_quant(const uint16_t *gate_up, int n_rows, int I, const int32_t *expert_off,
                        const int32_t *cnt_expert, int P, int fp8, void *act, float *act_scale)
{
    uint16_t *h = malloc(sizeof(uint16_t) * (size_t)(I > 0 ? I : 1));
    int S = I / 128;
    int n_groups = expert_off ? P : 1;
    for (int p = 0; p < n_groups; ++p) {
        int r0 = expert_off ? expert_off[p] : 0;
        int r1 = expert_off ? r0 + cnt_expert[p] : n_rows;
        if (r1 > n_rows) r1 = n_rows;
        for (int r = r0 < 0 ? 0 : r0; r < r1; ++r) {
            const uint16_t *row = gate_up + (size_t)r * 2 * I;
            if (fp8) {
                orc_silu_mul_row(row, I, h);
                orc_quantize_row(h, I, (uint8_t *)act + (size_t)r * I, act_scale + (size_t)r * S);
            } else {
                orc_silu_mul_row(row, I, (uint16_t *)act + (size_t)r * I);
            }
        }
    }
    free(h);
}
