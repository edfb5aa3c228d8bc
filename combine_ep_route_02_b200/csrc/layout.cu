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
// Three kernels, no inter-block waiting:
//   1. count:  one block per tile of LAYOUT_TILE tokens builds the tile's
//              per-expert histogram in shared memory, writes in_rank for its
//              tokens and the tile's per-rank token counts.
//   2. scan:   one warp per expert column turns the tile histograms into
//              exclusive per-tile offsets (in place) and the expert totals;
//              extra warps total the per-rank token counts.
//   3. slot:   one block per tile scans the expert totals, then each warp
//              orders its share of the tile's (t, j) pairs with match_any so
//              that rows inside an expert follow (t, j) order.
// Shared-memory atomics only count; no order is decided by an atomic.
#include "ep_device.cuh"
#include "ep_internal.h"

namespace ep {

namespace {

constexpr int BAD_EXPERT = 1;
constexpr int BAD_REPLICA = 2;

EP_DEV int phys_expert(const LayoutArgs &a, int t, int j, int &bad)
{
    const int e = a.topk_idx[(size_t)t * a.k + j];
    if ((unsigned)e >= (unsigned)a.E) {
        bad |= BAD_EXPERT;
        return -1;
    }
    if (a.phys_of == nullptr) return e;
    const int n = a.n_rep[e];
    if (n < 1 || n > a.max_rep) {
        bad |= BAD_REPLICA;
        return -1;
    }
    const int p = a.phys_of[(size_t)e * a.max_rep + (t % n)];
    if ((unsigned)p >= (unsigned)a.P) {
        bad |= BAD_REPLICA;
        return -1;
    }
    return p;
}

__global__ void __launch_bounds__(LAYOUT_THREADS) layout_count_kernel(LayoutArgs a)
{
    extern __shared__ int smem[];
    int *hist = smem;          // [P]
    int *tokr = hist + a.P;    // [R]
    int *pp = tokr + a.R;      // [LAYOUT_TILE * k]

    const int tile = blockIdx.x;
    const int t0 = tile * LAYOUT_TILE;
    const int nt = min(LAYOUT_TILE, a.T - t0);
    const int npairs = nt * a.k;

    for (int i = threadIdx.x; i < a.P; i += blockDim.x) hist[i] = 0;
    for (int i = threadIdx.x; i < a.R; i += blockDim.x) tokr[i] = 0;
    __syncthreads();

    int bad = 0;
    for (int i = threadIdx.x; i < npairs; i += blockDim.x) {
        const int p = phys_expert(a, t0 + i / a.k, i % a.k, bad);
        pp[i] = p;
        if (p >= 0) atomicAdd(&hist[p], 1);
    }
    if (bad && a.dev_status != nullptr) atomicOr(a.dev_status, bad);
    __syncthreads();

    const int epr = a.P / a.R;
    for (int i = threadIdx.x; i < nt * a.R; i += blockDim.x) {
        const int tl = i / a.R, r = i - tl * a.R;
        int hit = 0;
        for (int j = 0; j < a.k; ++j) {
            const int p = pp[tl * a.k + j];
            hit |= (p >= 0 && p / epr == r);
        }
        a.in_rank[(size_t)(t0 + tl) * a.R + r] = (uint8_t)hit;
        if (hit) atomicAdd(&tokr[r], 1);
    }
    __syncthreads();

    for (int i = threadIdx.x; i < a.P; i += blockDim.x) a.tile_cnt[(size_t)tile * a.P + i] = hist[i];
    for (int i = threadIdx.x; i < a.R; i += blockDim.x) a.tile_tok[(size_t)tile * a.R + i] = tokr[i];
}

// warp per column: columns [0, P) are experts, [P, P+R) are ranks
__global__ void __launch_bounds__(LAYOUT_THREADS) layout_scan_kernel(LayoutArgs a, int NT)
{
    const int lane = threadIdx.x & 31;
    const int col = blockIdx.x * LAYOUT_WARPS + (threadIdx.x >> 5);
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

// exclusive scan of n ints held in shared memory (n <= MAX_PHYS), in place;
// returns the total.  Every thread of the block must call it.
__device__ int block_exclusive_scan(int *v, int n, int *warp_tot)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int per = (n + LAYOUT_THREADS - 1) / LAYOUT_THREADS;
    const int lo = min(n, threadIdx.x * per), hi = min(n, lo + per);
    int local = 0;
    for (int i = lo; i < hi; ++i) local += v[i];
    const int incl = warp_inclusive_scan(local);
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const int wt = (lane < LAYOUT_WARPS) ? warp_tot[lane] : 0;
        const int wincl = warp_inclusive_scan(wt);
        if (lane < LAYOUT_WARPS) warp_tot[lane] = wincl - wt;
        if (lane == LAYOUT_WARPS - 1) warp_tot[LAYOUT_WARPS] = wincl;
    }
    __syncthreads();
    int run = warp_tot[warp] + incl - local;
    for (int i = lo; i < hi; ++i) {
        const int c = v[i];
        v[i] = run;
        run += c;
    }
    const int total = warp_tot[LAYOUT_WARPS];
    __syncthreads();
    return total;
}

__global__ void __launch_bounds__(LAYOUT_THREADS) layout_slot_kernel(LayoutArgs a)
{
    extern __shared__ int smem[];
    int *eoff = smem;                          // [P + 1]
    int *whist = eoff + a.P + 1;               // [LAYOUT_WARPS][P]
    int *pp = whist + LAYOUT_WARPS * a.P;      // [LAYOUT_TILE * k]
    __shared__ int warp_tot[LAYOUT_WARPS + 1];

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int tile = blockIdx.x;
    const int t0 = tile * LAYOUT_TILE;
    const int nt = min(LAYOUT_TILE, a.T - t0);
    const int npairs = nt * a.k;

    for (int i = threadIdx.x; i < a.P; i += blockDim.x) eoff[i] = a.cnt_expert[i];
    for (int i = threadIdx.x; i < LAYOUT_WARPS * a.P; i += blockDim.x) whist[i] = 0;
    int bad = 0;  // already reported by the count kernel
    for (int i = threadIdx.x; i < npairs; i += blockDim.x)
        pp[i] = phys_expert(a, t0 + i / a.k, i % a.k, bad);
    __syncthreads();
    const int total = block_exclusive_scan(eoff, a.P, warp_tot);
    if (threadIdx.x == 0) eoff[a.P] = total;
    __syncthreads();

    if (tile == 0) {
        for (int i = threadIdx.x; i <= a.P; i += blockDim.x) a.expert_off[i] = eoff[i];
        const int epr = a.P / a.R;
        for (int r = threadIdx.x; r < a.R; r += blockDim.x) {
            a.rank_off[r] = eoff[r * epr];
            a.rows_rank[r] = eoff[(r + 1) * epr] - eoff[r * epr];
        }
        if (threadIdx.x == 0) a.rank_off[a.R] = total;
    }

    // each warp owns a contiguous share of the tile's pairs, in (t, j) order
    const int per = (npairs + LAYOUT_WARPS - 1) / LAYOUT_WARPS;
    const int lo = min(npairs, warp * per), hi = min(npairs, lo + per);
    int *my = whist + warp * a.P;
    for (int i = lo + lane; i < hi; i += 32) {
        const int p = pp[i];
        if (p >= 0) atomicAdd(&my[p], 1);
    }
    __syncthreads();
    // per expert: base row of each warp's share = expert start + tile offset
    // + rows of earlier warps in this tile
    for (int p = threadIdx.x; p < a.P; p += blockDim.x) {
        int base = eoff[p] + a.tile_cnt[(size_t)tile * a.P + p];
#pragma unroll
        for (int w = 0; w < LAYOUT_WARPS; ++w) {
            const int c = whist[w * a.P + p];
            whist[w * a.P + p] = base;
            base += c;
        }
    }
    __syncthreads();

    const unsigned lt = lanemask_lt();
    for (int c0 = lo; c0 < hi; c0 += 32) {  // warp-uniform bounds
        const int i = c0 + lane;
        const bool active = i < hi;
        const int p = active ? pp[i] : -2;
        const unsigned peers = __match_any_sync(FULL_MASK, p);
        const int pair = t0 * a.k + i;
        if (active) {
            if (p >= 0) {
                const int s = my[p] + __popc(peers & lt);
                a.slot[pair] = s;
                a.src[s] = pair;
            } else {
                a.slot[pair] = -1;
            }
        }
        __syncwarp();
        if (active && p >= 0 && (peers & lt) == 0) my[p] += __popc(peers);
        __syncwarp();
    }
}

__global__ void layout_empty_kernel(LayoutArgs a)
{
    for (int i = threadIdx.x; i < a.P; i += blockDim.x) a.cnt_expert[i] = 0;
    for (int i = threadIdx.x; i <= a.P; i += blockDim.x) a.expert_off[i] = 0;
    for (int i = threadIdx.x; i < a.R; i += blockDim.x) {
        a.rows_rank[i] = 0;
        a.tok_rank[i] = 0;
    }
    for (int i = threadIdx.x; i <= a.R; i += blockDim.x) a.rank_off[i] = 0;
}

}  // namespace

cudaError_t launch_layout(const LayoutArgs &a, cudaStream_t s)
{
    cudaError_t err;
    if (a.dev_status != nullptr) {
        err = cudaMemsetAsync(a.dev_status, 0, sizeof(int32_t), s);
        if (err != cudaSuccess) return err;
    }
    if (a.T == 0) {
        layout_empty_kernel<<<1, 256, 0, s>>>(a);
        return cudaGetLastError();
    }
    const int NT = layout_tiles(a.T);
    const size_t sm_count = sizeof(int) * ((size_t)a.P + a.R + (size_t)LAYOUT_TILE * a.k);
    const size_t sm_slot =
        sizeof(int) * ((size_t)a.P + 1 + (size_t)LAYOUT_WARPS * a.P + (size_t)LAYOUT_TILE * a.k);
    if (sm_slot > 48 * 1024 || sm_count > 48 * 1024) {  // opt in above 48 KB
        static volatile int attr_set[64] = {0};
        int dev = 0;
        cudaGetDevice(&dev);
        if (dev >= 64 || !attr_set[dev]) {
            cudaFuncSetAttribute(layout_count_kernel,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
            cudaFuncSetAttribute(layout_slot_kernel,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
            if (dev < 64) attr_set[dev] = 1;
        }
    }
    layout_count_kernel<<<NT, LAYOUT_THREADS, sm_count, s>>>(a);
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
    const int cols = a.P + a.R;
    layout_scan_kernel<<<(cols + LAYOUT_WARPS - 1) / LAYOUT_WARPS, LAYOUT_THREADS, 0, s>>>(a, NT);
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
    layout_slot_kernel<<<NT, LAYOUT_THREADS, sm_slot, s>>>(a);
    return cudaGetLastError();
}

}  // namespace ep
