// Sigmoid-gated, group-limited top-k routing kernel (device code in
// route_impl.cuh): one warp per token, persistent grid.
#include "route_impl.cuh"

namespace ep {

namespace {

using namespace route_impl;

template <int EPL>
__global__ void __launch_bounds__(256, EPL <= 8 ? 4 : 1)
route_kernel(const float *__restrict__ logits, const float *__restrict__ bias, int T, int E,
             int G, int Kg, int k, float scale, int renorm, int vec4,
             int32_t *__restrict__ topk_idx, float *__restrict__ topk_w)
{
    pdl_launch_dependents();
    __shared__ double tab[64];
    load_exp_table(tab);
    __syncthreads();
    pdl_wait();
    const int warps = gridDim.x * (blockDim.x >> 5);
    route_tokens<EPL>(logits, bias, T, E, G, Kg, k, scale, renorm, vec4, topk_idx, topk_w, tab,
                      blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5), warps);
}

template <int EPL>
cudaError_t launch_epl(const RouteArgs &a, int vec4, cudaStream_t s)
{
    // persistent warps: one wave of resident blocks, each warp looping over
    // tokens, so no partly filled last wave
    const int warps_per_block = 8;
    int blocks = (a.T + warps_per_block - 1) / warps_per_block;
    static volatile int occ[64][6] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    const int slot = EPL == 1 ? 0 : EPL == 2 ? 1 : EPL == 4 ? 2 : EPL == 8 ? 3 : EPL == 16 ? 4 : 5;
    int per_sm = dev < 64 ? occ[dev][slot] : 0;
    if (per_sm <= 0) {
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, route_kernel<EPL>, 256, 0);
        if (per_sm <= 0) per_sm = 1;
        if (dev < 64) occ[dev][slot] = per_sm;
    }
    const int cap = device_sm_count() * per_sm;
    if (blocks > cap) blocks = cap;
    return launch_pdl(route_kernel<EPL>, dim3(blocks), dim3(warps_per_block * 32), 0, s, a.logits,
                      a.bias, a.T, a.E, a.G, a.Kg, a.k, a.scale, a.renorm, vec4, a.topk_idx,
                      a.topk_w);
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
