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
    const float r = __fmaf_rn(-q0, scale, x);
    // scale > 0, so the quotient carries the sign of x; the correction
    // would turn x = -0 into +0 (r = +0, then +0 + -0 = +0)
    return copysignf(__fmaf_rn(r, rcp, q0), x);
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

EP_DEV uint32_t quant4(const float *v, float scale, float rcp, bool fast)
{
    // q = e4m3(fp32(x / scale))
    float q[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) q[i] = fast ? div_by_scale(v[i], scale, rcp) : __fdiv_rn(v[i], scale);
    return pack_e4m3x2(q[0], q[1]) | (pack_e4m3x2(q[2], q[3]) << 16);
}

// Quantise one 16-element chunk (two 16-byte bf16 vectors).  The 8 lanes
// whose chunks form one 128-element block must call this together (xor
// shuffles over lane offsets 1, 2, 4); every lane of the warp must call it.
EP_DEV uint4 quant_chunk(uint4 lo, uint4 hi, float &scale_out)
{
    float v[16];
    v[0] = bf16_lo(lo.x);  v[1] = bf16_hi(lo.x);
    v[2] = bf16_lo(lo.y);  v[3] = bf16_hi(lo.y);
    v[4] = bf16_lo(lo.z);  v[5] = bf16_hi(lo.z);
    v[6] = bf16_lo(lo.w);  v[7] = bf16_hi(lo.w);
    v[8] = bf16_lo(hi.x);  v[9] = bf16_hi(hi.x);
    v[10] = bf16_lo(hi.y); v[11] = bf16_hi(hi.y);
    v[12] = bf16_lo(hi.z); v[13] = bf16_hi(hi.z);
    v[14] = bf16_lo(hi.w); v[15] = bf16_hi(hi.w);

    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(v[i]));
    amax = fmaxf(amax, __shfl_xor_sync(FULL_MASK, amax, 1));
    amax = fmaxf(amax, __shfl_xor_sync(FULL_MASK, amax, 2));
    amax = fmaxf(amax, __shfl_xor_sync(FULL_MASK, amax, 4));
    const float scale = __fdiv_rn(amax, 448.0f);
    scale_out = scale;

    uint4 q = make_uint4(0, 0, 0, 0);  // amax == 0: scale 0, zero bytes
    if (amax != 0.0f) {
        const bool fast = fast_div_ok(scale);
        const float rcp = fast ? __frcp_rn(scale) : 0.0f;
        q.x = quant4(v + 0, scale, rcp, fast);
        q.y = quant4(v + 4, scale, rcp, fast);
        q.z = quant4(v + 8, scale, rcp, fast);
        q.w = quant4(v + 12, scale, rcp, fast);
    }
    return q;
}

}  // namespace quant
}  // namespace ep
