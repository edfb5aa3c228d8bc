// Sigmoid-gated, group-limited top-k routing: one warp per token.
//
// DeepSeek group-limited routing (DeepSeek Open Infra day-4 summary, EPLB
// section) with plain top-k as its one-group special case (Perplexity blog,
// section "MoE Router").  Lane l holds experts [l*EPL, (l+1)*EPL); the group
// scores, the group choice and each of the k expert choices are warp-shuffle
// reductions, so no sort and no shared memory is needed.
#include <math.h>

#include "ep_device.cuh"
#include "ep_internal.h"

namespace ep {

namespace {

template <int EPL>
__global__ void __launch_bounds__(256)
route_kernel(const float *__restrict__ logits, const float *__restrict__ bias, int T, int E,
             int G, int Kg, int k, float scale, int renorm, int vec4,
             int32_t *__restrict__ topk_idx, float *__restrict__ topk_w)
{
    const int lane = threadIdx.x & 31;
    const int warps = gridDim.x * (blockDim.x >> 5);
    const int e0 = lane * EPL;
    const int gs = E / G;

    float b[EPL];
#pragma unroll
    for (int i = 0; i < EPL; ++i) b[i] = (bias != nullptr && e0 + i < E) ? bias[e0 + i] : 0.0f;

    for (int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); t < T; t += warps) {
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

        // s = fp32(1 / (1 + exp(-x))) evaluated in fp64; key = fp32(s + b)
        float s[EPL], key[EPL];
        unsigned excluded = 0;  // bit i: expert e0+i is not eligible
#pragma unroll
        for (int i = 0; i < EPL; ++i) {
            if (e0 + i < E) {
                s[i] = __double2float_rn(1.0 / (1.0 + exp(-(double)x[i])));
                key[i] = __fadd_rn(s[i], b[i]);
            } else {
                s[i] = 0.0f;
                key[i] = -INFINITY;
                excluded |= 1u << i;
            }
        }

        if (G > 1) {
            // group score = fp32 sum of the two largest keys in the group;
            // lane g keeps the score of group g
            float my_score = -INFINITY;
            for (int g = 0; g < G; ++g) {
                float a1 = -INFINITY, a2 = -INFINITY;
#pragma unroll
                for (int i = 0; i < EPL; ++i) {
                    const int e = e0 + i;
                    if (e < E && e / gs == g) {
                        const float v = key[i];
                        if (v > a1) {
                            a2 = a1;
                            a1 = v;
                        } else if (v > a2) {
                            a2 = v;
                        }
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
                if (lane == g) my_score = __fadd_rn(a1, a2);
            }
            // keep the Kg best groups, ties to the lower group id
            unsigned chosen = 0;
            for (int r = 0; r < Kg; ++r) {
                const bool cand = lane < G && !((chosen >> lane) & 1u);
                float v = cand ? my_score : -INFINITY;
                int id = cand ? lane : 0x7fffffff;
                warp_argmax(v, id);
                chosen |= 1u << id;
            }
#pragma unroll
            for (int i = 0; i < EPL; ++i) {
                const int e = e0 + i;
                if (e < E && !((chosen >> (e / gs)) & 1u)) excluded |= 1u << i;
            }
        }

        // k rounds of (key desc, index asc) arg-max over eligible experts
        unsigned taken = excluded;
        int sel_idx = 0;
        float sel_s = 0.0f;
        for (int r = 0; r < k; ++r) {
            float bv = -INFINITY;
            int bi = 0x7fffffff;
#pragma unroll
            for (int i = 0; i < EPL; ++i)
                if (!((taken >> i) & 1u) && beats(key[i], e0 + i, bv, bi)) {
                    bv = key[i];
                    bi = e0 + i;
                }
            warp_argmax(bv, bi);
            const int owner = bi / EPL;  // k <= eligible count: bi is a real expert
            float sv = 0.0f;
            if (lane == owner) {
#pragma unroll
                for (int i = 0; i < EPL; ++i)
                    if (e0 + i == bi) {
                        sv = s[i];
                        taken |= 1u << i;
                    }
            }
            sv = __shfl_sync(FULL_MASK, sv, owner);
            if (lane == r) {
                sel_idx = bi;
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
}

template <int EPL>
cudaError_t launch_epl(const RouteArgs &a, int vec4, cudaStream_t s)
{
    const int warps_per_block = 8;
    int blocks = (a.T + warps_per_block - 1) / warps_per_block;
    const int cap = device_sm_count() * 16;
    if (blocks > cap) blocks = cap;
    route_kernel<EPL><<<blocks, warps_per_block * 32, 0, s>>>(
        a.logits, a.bias, a.T, a.E, a.G, a.Kg, a.k, a.scale, a.renorm, vec4, a.topk_idx, a.topk_w);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_route(const RouteArgs &a, cudaStream_t s)
{
    if (a.T == 0) return cudaSuccess;
    const int vec4 = (a.E % 4 == 0) && ((reinterpret_cast<uintptr_t>(a.logits) & 15) == 0);
    if (a.E <= 32) return launch_epl<1>(a, vec4, s);
    if (a.E <= 64) return launch_epl<2>(a, vec4, s);
    if (a.E <= 128) return launch_epl<4>(a, vec4, s);
    if (a.E <= 256) return launch_epl<8>(a, vec4, s);
    if (a.E <= 512) return launch_epl<16>(a, vec4, s);
    return launch_epl<32>(a, vec4, s);
}

}  // namespace ep
