// Sigmoid-gated, group-limited top-k routing, device side: one warp per token.
// Included by the routing kernel and by the fused small-batch kernel.
//
// DeepSeek group-limited routing (DeepSeek Open Infra day-4 summary, EPLB
// section) with plain top-k as its one-group special case (Perplexity blog,
// section "MoE Router").  Lane l holds experts [l*EPL, (l+1)*EPL).
//
// Keys are compared as an order-preserving 32-bit image of the fp32 key.
// Keys are never -0.0 or NaN here (s >= 0, and s + b rounds an exact zero to
// +0), so the integer order equals the fp32 order.  The kept groups are the
// first topk_group in (score desc, id asc) order, found by ranking every
// group against all the others.  Each of the k experts is then one warp
// reduction: redux.sync max over the lanes' best keys, and the lowest lane
// holding that maximum (a ballot) owns the pick: lanes hold ascending index
// ranges and each lane's best is the lowest index of its largest key, so
// this is exactly the (key desc, index asc) order.
//
// When a group is a power-of-two number of whole lanes (E/G a multiple of
// EPL), each lane sits in one group and the group top-2 is a butterfly over
// that group's lanes only; otherwise a general loop over groups is used.
//
// The fp64 sigmoid uses a table-driven exp and a Newton reciprocal rather
// than the library exp and IEEE division: its fp64 value is within a few
// ulps of the exact one, far inside the 2^-47 relative distance from an fp32
// rounding midpoint below which another fp64 evaluation may round the other
// way, so the fp32 result is the same as any such evaluation's.
#pragma once

#include <math.h>

#include "ep_device.cuh"
#include "ep_internal.h"

namespace ep {
namespace route_impl {

// fp32 -> uint32 with the same order (for finite, non-NaN values; -0 and +0
// map to different images, which never matters for the keys used here).
EP_DEV uint32_t ordered(float f)
{
    const uint32_t b = __float_as_uint(f);
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

constexpr uint32_t NONE = 0u;  // below the image of every float, -inf included

// 2^(j/64) for j = 0..63, each correctly rounded to double
__constant__ double kExp2Frac[64] = {
    0x1.0000000000000p+0, 0x1.02c9a3e778061p+0, 0x1.059b0d3158574p+0, 0x1.0874518759bc8p+0,
    0x1.0b5586cf9890fp+0, 0x1.0e3ec32d3d1a2p+0, 0x1.11301d0125b51p+0, 0x1.1429aaea92de0p+0,
    0x1.172b83c7d517bp+0, 0x1.1a35beb6fcb75p+0, 0x1.1d4873168b9aap+0, 0x1.2063b88628cd6p+0,
    0x1.2387a6e756238p+0, 0x1.26b4565e27cddp+0, 0x1.29e9df51fdee1p+0, 0x1.2d285a6e4030bp+0,
    0x1.306fe0a31b715p+0, 0x1.33c08b26416ffp+0, 0x1.371a7373aa9cbp+0, 0x1.3a7db34e59ff7p+0,
    0x1.3dea64c123422p+0, 0x1.4160a21f72e2ap+0, 0x1.44e086061892dp+0, 0x1.486a2b5c13cd0p+0,
    0x1.4bfdad5362a27p+0, 0x1.4f9b2769d2ca7p+0, 0x1.5342b569d4f82p+0, 0x1.56f4736b527dap+0,
    0x1.5ab07dd485429p+0, 0x1.5e76f15ad2148p+0, 0x1.6247eb03a5585p+0, 0x1.6623882552225p+0,
    0x1.6a09e667f3bcdp+0, 0x1.6dfb23c651a2fp+0, 0x1.71f75e8ec5f74p+0, 0x1.75feb564267c9p+0,
    0x1.7a11473eb0187p+0, 0x1.7e2f336cf4e62p+0, 0x1.82589994cce13p+0, 0x1.868d99b4492edp+0,
    0x1.8ace5422aa0dbp+0, 0x1.8f1ae99157736p+0, 0x1.93737b0cdc5e5p+0, 0x1.97d829fde4e50p+0,
    0x1.9c49182a3f090p+0, 0x1.a0c667b5de565p+0, 0x1.a5503b23e255dp+0, 0x1.a9e6b5579fdbfp+0,
    0x1.ae89f995ad3adp+0, 0x1.b33a2b84f15fbp+0, 0x1.b7f76f2fb5e47p+0, 0x1.bcc1e904bc1d2p+0,
    0x1.c199bdd85529cp+0, 0x1.c67f12e57d14bp+0, 0x1.cb720dcef9069p+0, 0x1.d072d4a07897cp+0,
    0x1.d5818dcfba487p+0, 0x1.da9e603db3285p+0, 0x1.dfc97337b9b5fp+0, 0x1.e502ee78b3ff6p+0,
    0x1.ea4afa2a490dap+0, 0x1.efa1bee615a27p+0, 0x1.f50765b6e4540p+0, 0x1.fa7c1819e90d8p+0,
};

// exp(y) for -700 <= y <= 700 in fp64, table-driven after P. T. P. Tang,
// "Table-driven implementation of the exponential function in IEEE
// floating-point arithmetic", ACM TOMS 15(2), 1989: y = (64 m + j) ln2/64 + r
// with |r| <= ln2/128, exp(y) = 2^m * 2^(j/64) * (1 + p(r)), p the degree-6
// Taylor polynomial of e^r - 1 (truncation below 2^-64).  ln2/64 is split so
// that N * L1 is exact for |N| < 2^17.  Error: a few units in the last place.
EP_DEV double exp_table(double y, const double *tab)
{
    const double K = 0x1.71547652b82fep+6;   // 64 / ln 2
    const double L1 = 0x1.62e42fefa0000p-7;  // high 36 bits of ln2 / 64
    const double L2 = 0x1.cf79abc9e3b3ap-46; // ln2 / 64 - L1
    // N = y * K rounded to the nearest integer (ties to even): adding
    // 1.5 * 2^52 leaves N in the low bits of the sum, since |y K| < 2^51
    const double SHIFT = 0x1.8p52;
    const double big = __dadd_rn(__dmul_rn(y, K), SHIFT);
    const double Nd = __dsub_rn(big, SHIFT);
    const int N = __double2loint(big);
    double r = fma(-Nd, L1, y);
    r = fma(-Nd, L2, r);
    double p = fma(r, 1.0 / 720.0, 1.0 / 120.0);
    p = fma(r, p, 1.0 / 24.0);
    p = fma(r, p, 1.0 / 6.0);
    p = fma(r, p, 0.5);
    p = fma(r, p, 1.0);
    p = p * r;
    const double t = tab[N & 63];
    const double e = fma(t, p, t);
    return e * __hiloint2double((1023 + (N >> 6)) << 20, 0);
}

// ---- the exact sigmoid rounded once to fp32 -----------------------------
//
// sigmoid_fast evaluates 1 / (1 + e^-x) in fp64 to within a few fp64 ulps and
// rounds it to fp32; that is the correct rounding unless the fp64 value lies
// within 64 fp64 ulps (about 2^-46, relative) of an fp32 rounding midpoint,
// which sigmoid_fast reports in `near` (about one input in 2^22).  Those take
// sigmoid_exact: the same quantity in double-double arithmetic (Dekker's
// exact products and sums, error below 2^-95 relative) and a comparison with
// the midpoint.  No fp32 input has a sigmoid closer than 2^-100 to a
// midpoint, so the result is the exact value's rounding in every case.

// s = fp32(1 / (1 + exp(-x))) from an fp64 evaluation accurate to a few
// fp64 ulps (the reciprocal: a hardware estimate and two Newton steps).
EP_DEV float sigmoid_fast(float x, const double *tab, bool &near)
{
    double y = -(double)x;
    near = false;
    if (y > 700.0) return 0.0f;    // s < e^-700 rounds to +0 in fp32
    if (y < -700.0) y = -700.0;    // 1 + e^y rounds to 1 either way
    const double d = 1.0 + exp_table(y, tab);
    double z;
    asm("rcp.approx.ftz.f64 %0, %1;" : "=d"(z) : "d"(d));
    z = fma(z, fma(-d, z, 1.0), z);
    z = fma(z, fma(-d, z, 1.0), z);
    const float f = __double2float_rn(z);
    if (z >= 0x1p-126) {
        // fp32 normal: rounding looks at the low 29 of the 52 fraction bits;
        // 2^28 there is the midpoint
        const int lo = (int)((uint32_t)__double2loint(z) & 0x1FFFFFFFu) - (1 << 28);
        near = (unsigned)(lo + 64) <= 128u;
    } else {
        // fp32 subnormal (x below about -87): compare with the midpoint
        const double fd = (double)f;
        const double g = (double)__uint_as_float(z >= fd ? __float_as_uint(f) + 1u
                                                          : __float_as_uint(f) - 1u);
        near = fabs(z - 0.5 * (fd + g)) <= 0x1p-46 * z;
    }
    return f;
}

struct DD {
    double hi, lo;
};

// a + b exactly, as hi + lo (Knuth)
EP_DEV DD two_sum(double a, double b)
{
    const double s = __dadd_rn(a, b);
    const double bb = __dsub_rn(s, a);
    return {s, __dadd_rn(__dsub_rn(a, __dsub_rn(s, bb)), __dsub_rn(b, bb))};
}
// a + b exactly for |a| >= |b| (Dekker)
EP_DEV DD quick_two_sum(double a, double b)
{
    const double s = __dadd_rn(a, b);
    return {s, __dsub_rn(b, __dsub_rn(s, a))};
}
EP_DEV DD dd_add(DD a, DD b)
{
    const DD s = two_sum(a.hi, b.hi);
    const DD t = two_sum(a.lo, b.lo);
    DD v = quick_two_sum(s.hi, __dadd_rn(s.lo, t.hi));
    return quick_two_sum(v.hi, __dadd_rn(t.lo, v.lo));
}
EP_DEV DD dd_mul(DD a, DD b)
{
    const double p = __dmul_rn(a.hi, b.hi);
    const double e = __fma_rn(a.hi, b.hi, -p);  // a.hi * b.hi - p, exact
    const double t = __fma_rn(a.hi, b.lo, __fma_rn(a.lo, b.hi, e));
    return quick_two_sum(p, t);
}

// The exact sigmoid rounded to fp32, for the inputs sigmoid_fast flags.
// e^y with y = -x: y = N ln2 + r (ln2 in three parts, the first with 11
// trailing zero bits so N times it is exact), e^r = (e^(r/256))^256 with
// e^(r/256) - 1 from its Taylor series to degree 10 (remainder below 2^-104)
// and eight squarings of 1 + p as p <- 2p + p^2; then 1 / (1 + e^y) by a
// Newton step on the fp64 quotient, and the side of the fp32 midpoint.
static __device__ __noinline__ float sigmoid_exact(float x)
{
    double y = -(double)x;
    if (y > 700.0) return 0.0f;
    if (y < -700.0) y = -700.0;
    const double L1 = 0x1.62e42fefa3800p-1, L2 = 0x1.ef35793c76730p-45,
                 L3 = 0x1.f97b57a079a19p-103;
    const double N = rint(__dmul_rn(y, 0x1.71547652b82fep+0));  // y / ln2, to an integer
    const double r_hi = __fma_rn(-N, L1, y);                    // exact
    DD r = dd_add({r_hi, 0.0}, {__dmul_rn(-N, L2), __fma_rn(-N, L2, __dmul_rn(N, L2))});
    r = dd_add(r, {__dmul_rn(-N, L3), 0.0});
    r.hi = __dmul_rn(r.hi, 0x1p-8);  // r / 256, exact
    r.lo = __dmul_rn(r.lo, 0x1p-8);
    // 1/n! as two doubles each (hi = nearest double, lo = the remainder)
    const DD c[11] = {{0.0, 0.0}, {1.0, 0.0}, {0.5, 0.0},
                      {0x1.5555555555555p-3, 0x1.5555555555555p-57},
                      {0x1.5555555555555p-5, 0x1.5555555555555p-59},
                      {0x1.1111111111111p-7, 0x1.1111111111111p-63},
                      {0x1.6c16c16c16c17p-10, -0x1.f49f49f49f49fp-65},
                      {0x1.a01a01a01a01ap-13, 0x1.a01a01a01a01ap-73},
                      {0x1.a01a01a01a01ap-16, 0x1.a01a01a01a01ap-76},
                      {0x1.71de3a556c734p-19, -0x1.c154f8ddc6c00p-73},
                      {0x1.27e4fb7789f5cp-22, 0x1.cbbc05b4fa99ap-76}};
    DD p = c[10];
    for (int n = 9; n >= 1; --n) p = dd_add(dd_mul(p, r), c[n]);
    p = dd_mul(p, r);  // e^(r/256) - 1
    for (int i = 0; i < 8; ++i) p = dd_add({__dmul_rn(p.hi, 2.0), __dmul_rn(p.lo, 2.0)}, dd_mul(p, p));
    DD e = dd_add({1.0, 0.0}, p);  // e^r
    const int n = (int)N;          // |N| <= 1010: scale by 2^N in two exact steps
    const double s1 = __hiloint2double((1023 + n / 2) << 20, 0);
    const double s2 = __hiloint2double((1023 + (n - n / 2)) << 20, 0);
    e.hi = __dmul_rn(__dmul_rn(e.hi, s1), s2);
    e.lo = __dmul_rn(__dmul_rn(e.lo, s1), s2);
    const DD d = dd_add({1.0, 0.0}, e);
    const double q = __ddiv_rn(1.0, d.hi);
    // 1 - d q, exact for the hi part, then the lo part's share
    const double res = __dsub_rn(__fma_rn(-d.hi, q, 1.0), __dmul_rn(d.lo, q));
    const DD s = quick_two_sum(q, __dmul_rn(res, q));
    const float lo32 = __double2float_rd(s.hi), hi32 = __double2float_ru(s.hi);
    if (lo32 == hi32) return lo32;
    const double mid = 0.5 * ((double)lo32 + (double)hi32);  // exact
    const double t = __dadd_rn(__dsub_rn(s.hi, mid), s.lo);
    if (t > 0.0) return hi32;
    if (t < 0.0) return lo32;
    return (__float_as_uint(lo32) & 1u) ? hi32 : lo32;  // a tie: to even (never met)
}

// The lane's best key and its expert: the first (lowest index) of the
// largest keys, by a tree of pairwise picks (the right half of a pair wins
// only with a strictly larger key), so the dependency chain is log2(EPL)
// steps long.  EPL is a power of two.
template <int EPL>
EP_DEV void lane_best(const uint32_t (&key)[EPL], int e0, uint32_t &best_k, int &best_i)
{
    uint32_t tk[EPL];
    int ti[EPL];
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
        tk[i] = key[i];
        ti[i] = e0 + i;
    }
#pragma unroll
    for (int w = EPL / 2; w >= 1; w >>= 1)
#pragma unroll
        for (int j = 0; j < w; ++j) {
            const bool right = tk[2 * j + 1] > tk[2 * j];
            tk[j] = right ? tk[2 * j + 1] : tk[2 * j];
            ti[j] = right ? ti[2 * j + 1] : ti[2 * j];
        }
    best_k = tk[0];
    best_i = ti[0];
}

// Bias and token-invariant group id of each expert a lane holds (lane l
// holds experts [l*EPL, (l+1)*EPL)); -1: no such expert.
template <int EPL>
EP_DEV void lane_experts(const float *__restrict__ bias, int E, int G, float (&b)[EPL],
                         int (&gid)[EPL])
{
    const int e0 = (threadIdx.x & 31) * EPL;
    const int gs = E / G;
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
        const bool v = e0 + i < E;
        b[i] = (bias != nullptr && v) ? bias[e0 + i] : 0.0f;
        gid[i] = v ? (e0 + i) / gs : -1;
    }
}

// Selection for token t from its sigmoids s (the lane layout above; 0 for
// experts past E): keys s + b, group scores and the kept groups, the k
// largest keys, the weights; writes row t of topk_idx and topk_w.
template <int EPL>
EP_DEV void select_topk(float (&s)[EPL], const float (&b)[EPL], const int (&gid)[EPL], int E,
                        int G, int Kg, int k, float scale, int renorm,
                        int32_t *__restrict__ topk_idx, float *__restrict__ topk_w, int t)
{
    const int lane = threadIdx.x & 31;
    const int e0 = lane * EPL;
    const int gs = E / G;
    // each lane lies inside one group when gs is a multiple of EPL; the
    // butterfly below also needs the group's lane count to be a power of two
    const int lpg = gs / EPL;
    const bool aligned = (gs % EPL) == 0 && (lpg & (lpg - 1)) == 0;
    const int lanes_per_group = aligned ? lpg : 0;
    const int my_group = (e0 < E) ? e0 / gs : -1;        // valid when aligned
    uint32_t key[EPL];
    uint32_t live = 0;  // bit i: expert e0+i exists and is still eligible
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
        if (e0 + i < E) {
            key[i] = ordered(__fadd_rn(__fadd_rn(s[i], b[i]), 0.0f));
            live |= 1u << i;
        } else {
            key[i] = NONE;
        }
    }

    if (G > 1) {
        // group score = fp32 sum of the two largest keys in the group; the
        // lane that holds group g's score (every lane of the group when
        // aligned, lane g otherwise)
        uint32_t my_score = NONE;
        int score_lane_step = 1;
        if (aligned) {
            float a1 = -INFINITY, a2 = -INFINITY;
#pragma unroll
            for (int i = 0; i < EPL; ++i) {
                if (!((live >> i) & 1u)) continue;
                const float v = __fadd_rn(s[i], b[i]);
                if (v > a1) {
                    a2 = a1;
                    a1 = v;
                } else if (v > a2) {
                    a2 = v;
                }
            }
            // butterfly over the lanes of this group (they are contiguous
            // and start at a multiple of lanes_per_group)
            for (int off = 1; off < lanes_per_group; off <<= 1) {
                const float o1 = __shfl_xor_sync(FULL_MASK, a1, off);
                const float o2 = __shfl_xor_sync(FULL_MASK, a2, off);
                const float n2 = (a1 >= o1) ? fmaxf(a2, o1) : fmaxf(a1, o2);
                a1 = fmaxf(a1, o1);
                a2 = n2;
            }
            if (my_group >= 0) my_score = ordered(__fadd_rn(__fadd_rn(a1, a2), 0.0f));
            score_lane_step = lanes_per_group;
        } else {
            for (int g = 0; g < G; ++g) {
                float a1 = -INFINITY, a2 = -INFINITY;
#pragma unroll
                for (int i = 0; i < EPL; ++i) {
                    if (gid[i] != g) continue;
                    const float v = __fadd_rn(s[i], b[i]);
                    if (v > a1) {
                        a2 = a1;
                        a1 = v;
                    } else if (v > a2) {
                        a2 = v;
                    }
                }
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) {
                    const float o1 = __shfl_xor_sync(FULL_MASK, a1, off);
                    const float o2 = __shfl_xor_sync(FULL_MASK, a2, off);
                    const float n2 = (a1 >= o1) ? fmaxf(a2, o1) : fmaxf(a1, o2);
                    a1 = fmaxf(a1, o1);
                    a2 = n2;
                }
                if (lane == g) my_score = ordered(__fadd_rn(__fadd_rn(a1, a2), 0.0f));
            }
        }
        // the Kg groups first in (score descending, id ascending) order:
        // lane g < G ranks group g against every group and keeps it when
        // fewer than Kg come before it (the same set as Kg successive
        // arg-max picks with ties to the lower id)
        const int gl = lane < G ? lane : 0;
        const uint32_t sc_mine = __shfl_sync(FULL_MASK, my_score, gl * score_lane_step);
        int before = 0;
        for (int g = 0; g < G; ++g) {
            const uint32_t sc = __shfl_sync(FULL_MASK, my_score, g * score_lane_step);
            before += (sc > sc_mine || (sc == sc_mine && g < gl)) ? 1 : 0;
        }
        const uint32_t chosen = __ballot_sync(FULL_MASK, lane < G && before < Kg);
        if (aligned) {
            // the lane's experts share one group
            if (my_group >= 0 && !((chosen >> my_group) & 1u))
#pragma unroll
                for (int i = 0; i < EPL; ++i) key[i] = NONE;
        } else {
#pragma unroll
            for (int i = 0; i < EPL; ++i)
                if (gid[i] >= 0 && !((chosen >> gid[i]) & 1u)) key[i] = NONE;
        }
    }

    // lane-local best: the first (lowest index) of the largest keys;
    // excluded and taken experts hold NONE, below every real key (a lane
    // whose keys are all NONE is never the owner of a pick)
    uint32_t best_k;
    int best_i;
    lane_best<EPL>(key, e0, best_k, best_i);

    int sel_idx = 0;
    float sel_s = 0.0f;
    for (int r = 0; r < k; ++r) {
        // the largest key; among equal ones the lowest lane holds the lowest
        // index (lanes own ascending index ranges), and its best_i is the
        // lowest index of that key in the lane
        const uint32_t kmax = __reduce_max_sync(FULL_MASK, best_k);
        const int owner = __ffs(__ballot_sync(FULL_MASK, best_k == kmax)) - 1;
        const int e = __shfl_sync(FULL_MASK, best_i, owner);
        // every lane runs the owner's update; only the owner keeps it (no
        // divergent branch inside the pick loop)
        const bool own = lane == owner;
        const int mine = best_i;
        float sv = 0.0f;
#pragma unroll
        for (int i = 0; i < EPL; ++i) {
            const bool hit = own && (e0 + i == mine);
            sv = hit ? s[i] : sv;
            key[i] = hit ? NONE : key[i];
        }
        uint32_t nk;
        int ni;
        lane_best<EPL>(key, e0, nk, ni);
        best_k = own ? nk : best_k;
        best_i = own ? ni : best_i;
        sv = __shfl_sync(FULL_MASK, sv, owner);
        if (lane == r) {
            sel_idx = e;
            sel_s = sv;
        }
    }

    float w = sel_s;
    if (renorm) {
        float sum = 0.0f;
        for (int j = 0; j < k; ++j) sum = __fadd_rn(sum, __shfl_sync(FULL_MASK, sel_s, j));
        if (sum != 0.0f) w = __fdiv_rn(w, sum);
    }
    w = __fmul_rn(w, scale);
    if (lane < k) {
        topk_idx[(size_t)t * k + lane] = sel_idx;
        topk_w[(size_t)t * k + lane] = w;
    }
}

// Routes tokens t_first, t_first + t_stride, ... < T with the calling warp.
// tab: the 2^(j/64) table in shared memory.
template <int EPL>
EP_DEV void route_tokens(const float *__restrict__ logits, const float *__restrict__ bias, int T,
                         int E, int G, int Kg, int k, float scale, int renorm, int vec4,
                         int32_t *__restrict__ topk_idx, float *__restrict__ topk_w,
                         const double *tab, int t_first, int t_stride)
{
    const int lane = threadIdx.x & 31;
    const int e0 = lane * EPL;
    float b[EPL];
    int gid[EPL];
    lane_experts<EPL>(bias, E, G, b, gid);

    for (int t = t_first; t < T; t += t_stride) {
        const float *row = logits + (size_t)t * E;
        float x[EPL];
        if (EPL % 4 == 0 && vec4) {
#pragma unroll
            for (int q = 0; q < EPL / 4; ++q) {
                // E % 4 == 0, so a quad is either wholly inside the row or not
                float4 v = (e0 + 4 * q < E)
                               ? __ldg(reinterpret_cast<const float4 *>(row + e0) + q)
                               : make_float4(0.f, 0.f, 0.f, 0.f);
                x[4 * q + 0] = v.x;
                x[4 * q + 1] = v.y;
                x[4 * q + 2] = v.z;
                x[4 * q + 3] = v.w;
            }
        } else {
#pragma unroll
            for (int i = 0; i < EPL; ++i) x[i] = (e0 + i < E) ? __ldg(row + e0 + i) : 0.0f;
        }

        // s = the exact sigmoid rounded to fp32
        float s[EPL];
        uint32_t near = 0;  // bit i: s[i] needs the exact evaluation
#pragma unroll
        for (int i = 0; i < EPL; ++i) {
            bool nr = false;
            s[i] = (e0 + i < E) ? sigmoid_fast(x[i], tab, nr) : 0.0f;
            near |= (uint32_t)nr << i;
        }
        if (__any_sync(FULL_MASK, near != 0)) {
#pragma unroll
            for (int i = 0; i < EPL; ++i)
                if ((near >> i) & 1u) s[i] = sigmoid_exact(x[i]);
        }
        select_topk<EPL>(s, b, gid, E, G, Kg, k, scale, renorm, topk_idx, topk_w, t);
    }
}


// copies the exp table into shared memory (all threads of the block call it)
EP_DEV void load_exp_table(double *tab)
{
    for (int i = threadIdx.x; i < 64; i += blockDim.x) tab[i] = kExp2Frac[i];
}

}  // namespace route_impl
}  // namespace ep
