// 1x128 block quantisation to e4m3, device side: shared by dispatch (token
// rows) and the expert activation (SiLU rows).
//
// Per 128-element block: amax = max |x|, scale = fp32(amax / 448), and
// q = e4m3_rn_satfinite(fp32(x / scale)); a block with amax == 0 gets scale 0
// and zero bytes (Perplexity blog, section "Quantization": one scale per
// 128-element activation vector, from its maximum absolute value).
#pragma once

#include "ep_device.cuh"

namespace ep {
namespace quant {

// fp32(x / scale), rounded to nearest even, from the block's shared
// reciprocal rcp = fp32(1 / scale): one product, then Markstein's correction
// step (P. Markstein, "Computation of elementary functions on the IBM RISC
// System/6000 processor", IBM J. Res. Dev. 34(1), 1990): the residual
// x - q0 * scale is exact in one FMA and q0 + residual * rcp rounds to the
// correctly rounded quotient.  Used only for normal scales with a normal
// reciprocal (see fast_div_ok); the exhaustive dispatch test checks every
// bf16 (x, amax) pair against the oracle's IEEE division.
EP_DEV float div_by_scale(float x, float scale, float rcp)
{
    const float q0 = __fmul_rn(x, rcp);
    // the residual with its sign flipped, q0 * scale - x (exact in one FMA);
    // adding its negation keeps the sign of a zero quotient: for x = -0 it
    // gives -0 + -0 = -0, where x - q0 * scale would give +0 + -0 = +0
    const float rn = __fmaf_rn(q0, scale, -x);
    return __fmaf_rn(-rn, rcp, q0);
}

// The correction is exact while the residual cannot underflow: for a
// quotient large enough to reach an e4m3 rounding point (>= 2^-11) the
// residual is about 2^-23 |x| >= 2^-34 scale, a normal number once
// scale >= 2^-90; smaller quotients encode to zero either way.  Tinier
// scales (amax below about 3.6e-25) take the IEEE division.
EP_DEV bool fast_div_ok(float scale)
{
    return scale >= 0x1p-90f && scale <= 0x1p125f;
}

// q = e4m3(fp32(x / scale)) for 16 values: FAST divides through the block's
// reciprocal (normal scales, see fast_div_ok), otherwise by IEEE division.
// The two are separate code paths so that neither is executed predicated
// beside the other.
template <bool FAST>
EP_DEV uint4 quant16(const float *v, float scale, float rcp)
{
    float q[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) q[i] = FAST ? div_by_scale(v[i], scale, rcp) : __fdiv_rn(v[i], scale);
    uint4 r;
    r.x = pack_e4m3x2(q[0], q[1]) | (pack_e4m3x2(q[2], q[3]) << 16);
    r.y = pack_e4m3x2(q[4], q[5]) | (pack_e4m3x2(q[6], q[7]) << 16);
    r.z = pack_e4m3x2(q[8], q[9]) | (pack_e4m3x2(q[10], q[11]) << 16);
    r.w = pack_e4m3x2(q[12], q[13]) | (pack_e4m3x2(q[14], q[15]) << 16);
    return r;
}

EP_DEV void unpack16(uint4 lo, uint4 hi, float *v)
{
    v[0] = bf16_lo(lo.x);  v[1] = bf16_hi(lo.x);
    v[2] = bf16_lo(lo.y);  v[3] = bf16_hi(lo.y);
    v[4] = bf16_lo(lo.z);  v[5] = bf16_hi(lo.z);
    v[6] = bf16_lo(lo.w);  v[7] = bf16_hi(lo.w);
    v[8] = bf16_lo(hi.x);  v[9] = bf16_hi(hi.x);
    v[10] = bf16_lo(hi.y); v[11] = bf16_hi(hi.y);
    v[12] = bf16_lo(hi.z); v[13] = bf16_hi(hi.z);
    v[14] = bf16_lo(hi.w); v[15] = bf16_hi(hi.w);
}

// out of line, values passed packed: only blocks with a tiny (or non-finite)
// scale take it
static __device__ __noinline__ uint4 quant16_ieee(uint4 lo, uint4 hi, float scale)
{
    float v[16];
    unpack16(lo, hi, v);
    return quant16<false>(v, scale, 0.0f);
}

// Quantise one 16-element chunk (two 16-byte bf16 vectors).  The 8 lanes
// whose chunks form one 128-element block must call this together (xor
// shuffles over lane offsets 1, 2, 4); every lane of the warp must call it.
EP_DEV uint4 quant_chunk(uint4 lo, uint4 hi, float &scale_out)
{
    float v[16];
    unpack16(lo, hi, v);

    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(v[i]));
    amax = fmaxf(amax, __shfl_xor_sync(FULL_MASK, amax, 1));
    amax = fmaxf(amax, __shfl_xor_sync(FULL_MASK, amax, 2));
    amax = fmaxf(amax, __shfl_xor_sync(FULL_MASK, amax, 4));
    const float scale = __fdiv_rn(amax, 448.0f);
    scale_out = scale;

    if (amax == 0.0f) return make_uint4(0, 0, 0, 0);  // scale 0, zero bytes
    if (fast_div_ok(scale)) return quant16<true>(v, scale, __frcp_rn(scale));
    return quant16_ieee(lo, hi, scale);  // scales below 2^-90 (or inf, NaN): rare
}

}  // namespace quant
}  // namespace ep
