// Dispatch layout: per-expert / per-rank counts, prefix sums and
// deterministic, atomic-free slot assignment.
//
// The DeepEP V2 dispatch handle hands num_recv_tokens_per_expert_list to the
// expert GEMM (news.hada.io DeepEP summary, section "Usage for training,
// prefill and decoding"); the Perplexity blog (sections "MoE Router" and
// "CUDA Graph") notes that dense dispatch/combine plans need per-expert
// aggregates and that kernels must read those counts rather than size work
// from buffer capacities.
//
// Kernels (no block ever waits for another block):
//   count:  one block per tile of tokens builds the tile's per-expert
//           histogram in shared memory, writes in_rank for its tokens, the
//           tile's per-rank token counts and the tile's status bits.
//   [scan]: only for more than LAYOUT_FUSED_MAX_TILES tiles: one warp per
//           expert column turns the tile histograms into exclusive per-tile
//           offsets (in place) and the expert totals.
//   slot:   one block per tile.  With few tiles it first sums, for every
//           expert, the histograms of the tiles before it and of all tiles;
//           then it scans the expert totals, and each warp orders its share
//           of the tile's (t, j) pairs with match_any so that rows inside an
//           expert follow (t, j) order.
// Shared-memory atomics only count; no order is decided by an atomic.
#include "layout_impl.cuh"

namespace ep {

namespace {

using namespace layout_impl;

template <int NTH>
__global__ void __launch_bounds__(NTH) layout_count_kernel(LayoutArgs a)
{
    extern __shared__ int smem[];
    __shared__ int bad_sh;
    pdl_launch_dependents();
    pdl_wait();
    count_tile(a, blockIdx.x, smem, &bad_sh);
}

constexpr int SCAN_THREADS = 256;
constexpr int SCAN_WARPS = SCAN_THREADS / 32;

// many tiles: warp per column, columns [0, P) are experts, [P, P+R) ranks
__global__ void __launch_bounds__(SCAN_THREADS) layout_scan_kernel(LayoutArgs a)
{
    pdl_launch_dependents();
    pdl_wait();
    const int NT = a.n_tiles;
    const int lane = threadIdx.x & 31;
    const int col = blockIdx.x * SCAN_WARPS + (threadIdx.x >> 5);
    if (col >= a.P + a.R) return;  // warp-uniform
    if (col < a.P) {
        int running = 0;
        for (int base = 0; base < NT; base += 32) {
            const int i = base + lane;
            const int v = (i < NT) ? a.tile_cnt[(size_t)i * a.P + col] : 0;
            const int incl = warp_inclusive_scan(v);
            if (i < NT) a.tile_cnt[(size_t)i * a.P + col] = running + incl - v;
            running += __shfl_sync(FULL_MASK, incl, 31);
        }
        if (lane == 0) a.cnt_expert[col] = running;
    } else {
        const int r = col - a.P;
        int sum = 0;
        for (int i = lane; i < NT; i += 32) sum += a.tile_tok[(size_t)i * a.R + r];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(FULL_MASK, sum, off);
        if (lane == 0) a.tok_rank[r] = sum;
    }
}

template <int NTH, bool FUSED>
__global__ void __launch_bounds__(NTH) layout_slot_kernel(LayoutArgs a)
{
    extern __shared__ int smem[];
    __shared__ int warp_tot[NTH / 32 + 1];
    pdl_launch_dependents();
    pdl_wait();
    slot_tile<NTH, FUSED>(a, blockIdx.x, smem, warp_tot);
}

__global__ void layout_empty_kernel(LayoutArgs a)
{
    pdl_launch_dependents();
    pdl_wait();
    for (int i = threadIdx.x; i < a.P; i += blockDim.x) a.cnt_expert[i] = 0;
    for (int i = threadIdx.x; i <= a.P; i += blockDim.x) a.expert_off[i] = 0;
    for (int i = threadIdx.x; i < a.R; i += blockDim.x) {
        a.rows_rank[i] = 0;
        a.tok_rank[i] = 0;
    }
    for (int i = threadIdx.x; i <= a.R; i += blockDim.x) a.rank_off[i] = 0;
    if (threadIdx.x == 0 && a.dev_status != nullptr) *a.dev_status = 0;
}

void opt_in_smem(const void *fn, size_t bytes)
{
    // dynamic plus the kernels' static shared memory (under 1 KB) above the
    // default 48 KB needs an opt-in
    if (bytes + 1024 > 48 * 1024)
        cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

// The count and slot kernels for blocks of NTH threads.
template <int NTH>
cudaError_t launch_tiles(const LayoutArgs &a, cudaStream_t s)
{
    cudaError_t err;
    const int NT = a.n_tiles;
    const size_t pairs = (size_t)a.tile_tokens * a.k;
    const size_t sm_count = sizeof(int) * count_smem_ints(a.P, a.R, a.tile_tokens, a.k);
    const size_t sm_slot =
        sizeof(int) * ((size_t)2 * a.P + 1 + (size_t)a.hist_warps * a.P + pairs);
    const bool fused = NT <= LAYOUT_FUSED_MAX_TILES;
    opt_in_smem((const void *)layout_count_kernel<NTH>, sm_count);
    opt_in_smem(fused ? (const void *)layout_slot_kernel<NTH, true>
                      : (const void *)layout_slot_kernel<NTH, false>,
                sm_slot);
    err = launch_pdl(layout_count_kernel<NTH>, dim3(NT), dim3(NTH), sm_count, s, a);
    if (err != cudaSuccess) return err;
    if (fused)
        return launch_pdl(layout_slot_kernel<NTH, true>, dim3(NT), dim3(NTH), sm_slot, s, a);
    const int cols = a.P + a.R;
    err = launch_pdl(layout_scan_kernel, dim3((cols + SCAN_WARPS - 1) / SCAN_WARPS),
                     dim3(SCAN_THREADS), 0, s, a);
    if (err != cudaSuccess) return err;
    return launch_pdl(layout_slot_kernel<NTH, false>, dim3(NT), dim3(NTH), sm_slot, s, a);
}

}  // namespace

cudaError_t launch_layout(const LayoutArgs &a, cudaStream_t s)
{
    if (a.T == 0) return launch_pdl(layout_empty_kernel, dim3(1), dim3(256), 0, s, a);
    // Tiles of at most 512 pairs take blocks of 512 threads: every phase of
    // the two kernels ends in a block barrier, and with a small tile most of
    // 32 warps would only wait at them.  The slot kernel's ordering warps
    // (hist_warps) cannot outnumber the block's warps.
    if ((long long)a.tile_tokens * a.k <= 512) {
        LayoutArgs b = a;
        if (b.hist_warps > 512 / 32) b.hist_warps = 512 / 32;
        return launch_tiles<512>(b, s);
    }
    return launch_tiles<LAYOUT_THREADS>(a, s);
}

}  // namespace ep
