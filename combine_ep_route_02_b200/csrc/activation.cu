// Expert activation between the two grouped GEMMs of a gated-SiLU expert:
// h = silu(gate) * up for the rows the routing counts say are filled, then
// 1x128 block quantisation of h to e4m3 for the second GEMM.
//
// The Perplexity blog (section "Quantization") describes this kernel: the
// SiLU has to work under CUDA graphs, with block quantisation and with a
// token count that only the routing knows, so a fixed number of persistent
// blocks read the per-expert counts on the device and share out the filled
// rows among themselves instead of sizing the launch from the buffer.
//
// Arithmetic (exact, so the result does not depend on the schedule):
//   s = bf16(silu(g)), silu(g) = g / (1 + e^-g) correctly rounded
//   h = bf16(fp32(s * u))
//   then the dispatch quantiser on h (quant.cuh).
// The correctly rounded SiLU takes an fp32 evaluation (expf and a fast
// divide, a few fp32 ulps of error) and rounds it to bf16 unless the fp32
// value lies within 64 fp32 ulps of a bf16 rounding midpoint, or g is
// outside the range where that error bound holds; those inputs take an fp64
// evaluation.  Every one of the 65,536 bf16 inputs is checked against the
// oracle on the GPU.
//
// Mapping: the filled rows are numbered v = 0 .. V-1 in expert order (V = sum
// of the counts); a thread owns a 16-element chunk of one output row (two
// 16-byte loads of gate, two of up, one 16-byte store of e4m3), and the 8
// lanes of a 128-element block reduce its amax with shuffles.  Each block
// keeps the counts' prefix sum in shared memory and finds a chunk's expert
// by binary search.
#include "ep_device.cuh"
#include "ep_internal.h"
#include "quant.cuh"

namespace ep {

namespace {

constexpr int ACT_THREADS = 256;

// bf16 value of silu(g) in the slow cases: NaN, -inf, tiny |g|, g < -80, or
// an fp32 result too close to a bf16 midpoint.
__device__ __noinline__ float silu_bf16_slow(float g)
{
    if (g != g) return g;
    if (g == -INFINITY) return -0.0f;
    if (fabsf(g) < 0x1p-100f) {
        // silu(g) - g/2 = g tanh(g/2) / 2 > 0, far below fp32 and fp64
        // resolution here, and g/2 (exact in fp32) can be a bf16 midpoint:
        // the exact value lies just above g/2, so a tie rounds toward +inf
        // (up in magnitude for g > 0, down for g < 0).
        uint32_t u = __float_as_uint(g * 0.5f);
        u += (u >> 31) ? 0x7FFFu : 0x8000u;
        return __uint_as_float(u & 0xFFFF0000u);
    }
    const double x = (double)g;
    const double v = x / (1.0 + exp(-x));
    return __bfloat162float(__double2bfloat16(v));
}

EP_DEV float silu_bf16(float g)
{
    // fast range: e^-g stays below 2^126 (the fast divide's range) and the
    // quotient stays a normal fp32 number; NaN fails the first comparison
    if (g >= -80.0f && fabsf(g) >= 0x1p-60f) {
        const float s = __fdividef(g, 1.0f + expf(-g));
        const uint32_t u = __float_as_uint(s);
        // the 16 bits that bf16 rounding drops; 0x8000 is the midpoint
        if ((u & 0xFFFFu) - (0x8000u - 64u) > 128u) return bf16_lo(pack_bf16x2(s, 0.0f));
    }
    return silu_bf16_slow(g);
}

// h for the 8 elements of one 16-byte gate vector and one 16-byte up vector
EP_DEV uint4 silu_mul8(uint4 g, uint4 u)
{
    const uint32_t gp[4] = {g.x, g.y, g.z, g.w};
    const uint32_t up[4] = {u.x, u.y, u.z, u.w};
    uint32_t h[4];
#pragma unroll
    for (int m = 0; m < 4; ++m) {
        const float lo = __fmul_rn(silu_bf16(bf16_lo(gp[m])), bf16_lo(up[m]));
        const float hi = __fmul_rn(silu_bf16(bf16_hi(gp[m])), bf16_hi(up[m]));
        h[m] = pack_bf16x2(lo, hi);
    }
    return make_uint4(h[0], h[1], h[2], h[3]);
}

// Filled row number v -> buffer row: the last expert p with cum[p] <= v
// (experts with no rows share their cum value with the next one and are
// skipped by taking the last).
EP_DEV int filled_row(const int *cum, const int *eoff, int P, int v)
{
    int lo = 0, hi = P;  // cum[lo] <= v < cum[hi]
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (cum[mid] <= v) lo = mid;
        else hi = mid;
    }
    return eoff[lo] + (v - cum[lo]);
}

template <bool FP8>
__global__ void __launch_bounds__(ACT_THREADS)
silu_mul_kernel(const uint16_t *__restrict__ gate_up, int n_rows, int I,
                const int32_t *__restrict__ expert_off, const int32_t *__restrict__ cnt_expert,
                int P, void *__restrict__ act, float *__restrict__ act_scale)
{
    extern __shared__ int sm[];
    int *cum = sm;            // [P + 1]  prefix sum of the counts
    int *eoff = sm + P + 1;   // [P]      first buffer row of each expert
    __shared__ int warp_tot[ACT_THREADS / 32 + 1];
    pdl_launch_dependents();
    pdl_wait();

    int V = n_rows;
    if (expert_off != nullptr) {
        const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
        // block-wide exclusive scan of the counts, ACT_THREADS at a time
        int carry = 0;
        for (int base = 0; base < P; base += ACT_THREADS) {
            const int p = base + threadIdx.x;
            const int c = p < P ? cnt_expert[p] : 0;
            if (p < P) eoff[p] = expert_off[p];
            const int incl = warp_inclusive_scan(c);
            if (lane == 31) warp_tot[warp] = incl;
            __syncthreads();
            if (warp == 0) {
                const int wt = lane < ACT_THREADS / 32 ? warp_tot[lane] : 0;
                const int wi = warp_inclusive_scan(wt);
                if (lane < ACT_THREADS / 32) warp_tot[lane] = wi - wt;
                if (lane == ACT_THREADS / 32 - 1) warp_tot[ACT_THREADS / 32] = wi;
            }
            __syncthreads();
            if (p < P) cum[p] = carry + warp_tot[warp] + incl - c;
            carry += warp_tot[ACT_THREADS / 32];
            __syncthreads();
        }
        if (threadIdx.x == 0) cum[P] = carry;
        __syncthreads();
        V = min(carry, n_rows);
    }

    const int cpr = I >> 4;        // 16-element chunks per output row (multiple of 8)
    const int S = I >> 7;
    const long long total = (long long)V * cpr;
    const long long stride = (long long)gridDim.x * ACT_THREADS;
    // block-uniform loop bound so every lane reaches the shuffles; total is
    // a multiple of 8, so a lane octet is all active or all idle
    ChunkWalk it((long long)blockIdx.x * ACT_THREADS + threadIdx.x, stride, cpr);
    for (long long base = (long long)blockIdx.x * ACT_THREADS; base < total;
         base += stride, it.next()) {
        bool active = base + threadIdx.x < total;
        const int c = it.c;
        int row = 0;
        uint4 g0 = make_uint4(0, 0, 0, 0), g1 = g0, u0 = g0, u1 = g0;
        if (active) {
            row = expert_off != nullptr ? filled_row(cum, eoff, P, it.t) : it.t;
            active = (unsigned)row < (unsigned)n_rows;  // offsets beyond the buffer: skipped
        }
        if (active) {
            const uint16_t *gp = gate_up + (size_t)row * 2 * I + (size_t)c * 16;
            g0 = ld_stream(gp);
            g1 = ld_stream(gp + 8);
            u0 = ld_stream(gp + I);
            u1 = ld_stream(gp + I + 8);
        }
        const uint4 h0 = silu_mul8(g0, u0);
        const uint4 h1 = silu_mul8(g1, u1);
        if (FP8) {
            float scale;
            const uint4 q = quant::quant_chunk(h0, h1, scale);
            if (active) {
                st_stream(static_cast<uint8_t *>(act) + (size_t)row * I + (size_t)c * 16, q);
                if ((c & 7) == 0) st_stream_f32(act_scale + (size_t)row * S + (c >> 3), scale);
            }
        } else if (active) {
            uint16_t *o = static_cast<uint16_t *>(act) + (size_t)row * I + (size_t)c * 16;
            st_stream(o, h0);
            st_stream(o + 8, h1);
        }
    }
}

size_t act_smem_bytes(int P) { return sizeof(int) * (size_t)(2 * P + 1); }

}  // namespace

int activation_blocks_per_sm()
{
    int n = 0;
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, silu_mul_kernel<true>, ACT_THREADS,
                                                  act_smem_bytes(256));
    return n > 0 ? n : 1;
}

cudaError_t launch_activation(const ActivationArgs &a, cudaStream_t s)
{
    if (a.n_rows == 0) return cudaSuccess;
    const int P = a.expert_off != nullptr ? a.P : 0;
    const size_t smem = act_smem_bytes(P);
    const void *fn = a.fp8 ? (const void *)silu_mul_kernel<true> : (const void *)silu_mul_kernel<false>;
    if (smem > 48 * 1024) cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    // without counts the work is known on the host: no more blocks than chunks
    long long blocks = a.grid;
    if (a.expert_off == nullptr) {
        const long long chunks = (long long)a.n_rows * (a.I / 16);
        const long long need = (chunks + ACT_THREADS - 1) / ACT_THREADS;
        if (need < blocks) blocks = need;
    }
    if (a.fp8)
        return launch_pdl(silu_mul_kernel<true>, dim3((int)blocks), dim3(ACT_THREADS), smem, s,
                          static_cast<const uint16_t *>(a.gate_up), a.n_rows, a.I, a.expert_off,
                          a.cnt_expert, P, a.act, a.act_scale);
    return launch_pdl(silu_mul_kernel<false>, dim3((int)blocks), dim3(ACT_THREADS), smem, s,
                      static_cast<const uint16_t *>(a.gate_up), a.n_rows, a.I, a.expert_off,
                      a.cnt_expert, P, a.act, a.act_scale);
}

}  // namespace ep
