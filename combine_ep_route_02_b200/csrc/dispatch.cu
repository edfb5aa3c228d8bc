// Dispatch: permute token rows into rank-major, expert-contiguous receive rows,
// optionally quantising each row once to e4m3 with 1x128 block scales before
// writing its k copies.
//
// Per-128-element activation scales computed on the fly from the block's
// maximum absolute value (Perplexity blog, section "Quantization"); FP8
// dispatch with BF16 combine (DeepEP V2 summary, section "Performance").
//
// Mapping: a thread owns a 16-element chunk of a row (32 B of bf16 in, 16 B of
// e4m3 out); the 8 consecutive lanes that own one 128-element block reduce its
// amax with three xor-shuffles.  The row is read once and its quantised bytes
// are stored k times with 16-byte evict-first stores, so the k-fold write
// amplification costs no extra reads or arithmetic.
#include "ep_device.cuh"
#include "ep_internal.h"

namespace ep {

namespace {

constexpr int DISPATCH_THREADS = 256;

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

__global__ void __launch_bounds__(DISPATCH_THREADS)
dispatch_fp8_kernel(const uint16_t *__restrict__ x, int T, int H, int k,
                    const int32_t *__restrict__ slot, uint8_t *__restrict__ recv_x,
                    float *__restrict__ recv_scale, int n_rows)
{
    const int cpr = H >> 4;  // 16-element chunks per row (a multiple of 8)
    const int S = H >> 7;
    const long long total = (long long)T * cpr;
    const long long stride = (long long)gridDim.x * DISPATCH_THREADS;
    // the loop bound is block-uniform so every lane reaches the shuffles;
    // total is a multiple of 8, so a lane octet is all active or all idle
    const long long g0 = (long long)blockIdx.x * DISPATCH_THREADS + threadIdx.x;
    ChunkWalk it(g0, stride, cpr);
    for (long long base = (long long)blockIdx.x * DISPATCH_THREADS; base < total;
         base += stride, it.next()) {
        const bool active = it.t < T;
        const int t = it.t, c = it.c;
        uint4 lo = make_uint4(0, 0, 0, 0), hi = make_uint4(0, 0, 0, 0);
        if (active) {
            const uint16_t *p = x + (size_t)t * H + (size_t)c * 16;
            lo = ld_stream(p);
            hi = ld_stream(p + 8);
        }
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

        uint4 q = make_uint4(0, 0, 0, 0);  // amax == 0: scale 0, zero bytes
        if (amax != 0.0f) {
            const bool fast = fast_div_ok(scale);
            const float rcp = fast ? __frcp_rn(scale) : 0.0f;
            q.x = quant4(v + 0, scale, rcp, fast);
            q.y = quant4(v + 4, scale, rcp, fast);
            q.z = quant4(v + 8, scale, rcp, fast);
            q.w = quant4(v + 12, scale, rcp, fast);
        }
        if (active) {
            const int32_t *sl = slot + (size_t)t * k;
            for (int j = 0; j < k; ++j) {
                const int s = __ldg(sl + j);
                if ((unsigned)s < (unsigned)n_rows) {
                    st_stream(recv_x + (size_t)s * H + (size_t)c * 16, q);
                    if ((c & 7) == 0) st_stream_f32(recv_scale + (size_t)s * S + (c >> 3), scale);
                }
            }
        }
    }
}

__global__ void __launch_bounds__(DISPATCH_THREADS)
dispatch_bf16_kernel(const uint16_t *__restrict__ x, int T, int H, int k,
                     const int32_t *__restrict__ slot, uint16_t *__restrict__ recv_x, int n_rows)
{
    const int cpr = H >> 3;  // 8-element (16-byte) chunks per row
    const long long total = (long long)T * cpr;
    const long long g0 = (long long)blockIdx.x * DISPATCH_THREADS + threadIdx.x;
    if (g0 >= total) return;
    ChunkWalk it(g0, (long long)gridDim.x * DISPATCH_THREADS, cpr);
    for (; it.t < T; it.next()) {
        const int t = it.t, c = it.c;
        const uint4 v = ld_stream(x + (size_t)t * H + (size_t)c * 8);
        const int32_t *sl = slot + (size_t)t * k;
        for (int j = 0; j < k; ++j) {
            const int s = __ldg(sl + j);
            if ((unsigned)s < (unsigned)n_rows) st_stream(recv_x + (size_t)s * H + (size_t)c * 8, v);
        }
    }
}

}  // namespace

int dispatch_blocks_per_sm(int fp8)
{
    int n = 0;
    if (fp8)
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, dispatch_fp8_kernel, DISPATCH_THREADS, 0);
    else
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, dispatch_bf16_kernel, DISPATCH_THREADS, 0);
    return n > 0 ? n : 1;
}

cudaError_t launch_dispatch(const DispatchArgs &a, cudaStream_t s)
{
    if (a.T == 0) return cudaSuccess;
    const long long chunks = (long long)a.T * (a.fp8 ? a.H / 16 : a.H / 8);
    long long blocks = (chunks + DISPATCH_THREADS - 1) / DISPATCH_THREADS;
    if (blocks > a.grid) blocks = a.grid;
    const int n_rows = a.T * a.k;
    if (a.fp8)
        dispatch_fp8_kernel<<<(int)blocks, DISPATCH_THREADS, 0, s>>>(
            static_cast<const uint16_t *>(a.x), a.T, a.H, a.k, a.slot,
            static_cast<uint8_t *>(a.recv_x), a.recv_scale, n_rows);
    else
        dispatch_bf16_kernel<<<(int)blocks, DISPATCH_THREADS, 0, s>>>(
            static_cast<const uint16_t *>(a.x), a.T, a.H, a.k, a.slot,
            static_cast<uint16_t *>(a.recv_x), n_rows);
    return cudaGetLastError();
}

}  // namespace ep
