// Routing and dispatch layout of a small batch in one kernel.
//
// For decode-sized batches every step of the path is bound by launch and
// dependency latency, not bandwidth; the DeepEP V2 summary (section "Usage
// for training, prefill and decoding") and the Perplexity blog (section
// "CUDA Graph") both treat that case separately.  Here the routing warps of
// all blocks first write their tokens' top-k; each block then counts itself
// done on a counter (writes, __threadfence, atomicAdd), and the block that
// finds itself last lays out the whole batch as a single tile.  No block ever
// waits for another: the last block only does extra work.
#include "layout_impl.cuh"
#include "route_impl.cuh"

namespace ep {

namespace {

// shared memory of the last block: the count / slot phase tables, then what
// the count phase hands to the slot phase (the pair list, the expert and
// rank counts, the status bits), past the end of the slot phase's tables
#define SMALL_SMEM_READY_OFFSET(a) \
    (2 * (a).P + 1 + (a).hist_warps * (a).P + (a).T * (a).k)

template <int EPL>
__global__ void __launch_bounds__(256)
route_layout_small_kernel(RouteArgs r, LayoutArgs a, int vec4, int *done)
{
    extern __shared__ int smem[];
    __shared__ double tab[64];
    __shared__ int warp_tot[256 / 32 + 1];
    __shared__ int is_last, bad_sh;

    pdl_launch_dependents();
    route_impl::load_exp_table(tab);
    __syncthreads();
    pdl_wait();
    route_impl::route_tokens<EPL>(r.logits, r.bias, r.T, r.E, r.G, r.Kg, r.k, r.scale, r.renorm,
                                  vec4, r.topk_idx, r.topk_w, tab,
                                  blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5),
                                  gridDim.x * (blockDim.x >> 5));
    __threadfence();  // this block's top-k is visible before it counts itself done
    __syncthreads();
    if (threadIdx.x == 0) is_last = atomicAdd(done, 1) == (int)gridDim.x - 1;
    __syncthreads();
    if (!is_last) return;
    __threadfence();  // every other block's top-k is visible to the last block
    // the whole batch is tile 0; the slot phase takes the pair list and the
    // counts from shared memory, copied out of its way first
    int *ready = smem + SMALL_SMEM_READY_OFFSET(a);
    layout_impl::count_tile(a, 0, smem, &bad_sh);
    const int npairs = a.T * a.k;
    for (int i = threadIdx.x; i < npairs; i += blockDim.x) ready[i] = smem[a.P + a.R + i];
    for (int i = threadIdx.x; i < a.P + a.R; i += blockDim.x) ready[npairs + i] = smem[i];
    if (threadIdx.x == 0) ready[npairs + a.P + a.R] = bad_sh;
    __syncthreads();
    layout_impl::slot_tile<256, true>(a, 0, smem, warp_tot, ready);
}

template <int EPL>
cudaError_t launch_small(const RouteArgs &r, const LayoutArgs &a, int vec4, int *done,
                         size_t smem, cudaStream_t s)
{
    cudaError_t e = cudaMemsetAsync(done, 0, sizeof(int), s);
    if (e != cudaSuccess) return e;
    // dynamic plus the kernel's static shared memory (under 1 KB) above the
    // default 48 KB needs an opt-in
    if (smem + 1024 > 48 * 1024)
        cudaFuncSetAttribute(route_layout_small_kernel<EPL>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    const int blocks = (r.T + 7) / 8;  // a warp per token: T <= SMALL_MAX_PAIRS
    return launch_pdl(route_layout_small_kernel<EPL>, dim3(blocks), dim3(256), smem, s, r, a,
                      vec4, done);
}

}  // namespace

bool small_route_layout_ok(int T, int k, int P)
{
    return T > 0 && (long long)T * k <= SMALL_MAX_PAIRS && P <= SMALL_MAX_PHYS;
}

cudaError_t launch_route_layout_small(const RouteArgs &r, LayoutArgs a, int *done,
                                      cudaStream_t s)
{
    // the whole batch is one tile laid out by one block of 256 threads
    a.tile_tokens = r.T;
    a.n_tiles = 1;
    a.hist_warps = layout_hist_warps(a.P) < 8 ? layout_hist_warps(a.P) : 8;
    const size_t pairs = (size_t)r.T * r.k;
    const size_t count_ints = layout_impl::count_smem_ints(a.P, a.R, r.T, r.k);
    const size_t slot_ints = (size_t)2 * a.P + 1 + (size_t)a.hist_warps * a.P + pairs;
    // tables of the larger phase, then the hand-over region (it starts at
    // slot_ints, beyond every count-phase table it is copied from)
    const size_t big = count_ints > slot_ints ? count_ints : slot_ints;
    const size_t smem = sizeof(int) * (big + pairs + a.P + a.R + 1);
    const int vec4 = (r.E % 4 == 0) && ((reinterpret_cast<uintptr_t>(r.logits) & 15) == 0);
    if (r.E <= 32) return launch_small<1>(r, a, vec4, done, smem, s);
    if (r.E <= 64) return launch_small<2>(r, a, vec4, done, smem, s);
    if (r.E <= 128) return launch_small<4>(r, a, vec4, done, smem, s);
    if (r.E <= 256) return launch_small<8>(r, a, vec4, done, smem, s);
    if (r.E <= 512) return launch_small<16>(r, a, vec4, done, smem, s);
    return launch_small<32>(r, a, vec4, done, smem, s);
}

}  // namespace ep
