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
    int *pp = tokr + a.R;      // [tile_tokens * k]
    __shared__ int bad_sh;

    pdl_launch_dependents();
    const int tile = blockIdx.x;
    const int t0 = tile * a.tile_tokens;
    const int nt = min(a.tile_tokens, a.T - t0);
    const int npairs = nt * a.k;

    for (int i = threadIdx.x; i < a.P; i += blockDim.x) hist[i] = 0;
    for (int i = threadIdx.x; i < a.R; i += blockDim.x) tokr[i] = 0;
    if (threadIdx.x == 0) bad_sh = 0;
    __syncthreads();
    pdl_wait();

    int bad = 0;
    for (int i = threadIdx.x; i < npairs; i += blockDim.x) {
        const int p = phys_expert(a, t0 + i / a.k, i % a.k, bad);
        pp[i] = p;
        if (p >= 0) atomicAdd(&hist[p], 1);
    }
    if (bad) atomicOr(&bad_sh, bad);
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
    if (threadIdx.x == 0) a.tile_bad[tile] = bad_sh;
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

template <bool FUSED>
__global__ void __launch_bounds__(LAYOUT_THREADS) layout_slot_kernel(LayoutArgs a)
{
    extern __shared__ int smem[];
    const int HW = a.hist_warps;
    int *eoff = smem;                          // [P + 1]  expert start rows
    int *toff = eoff + a.P + 1;                // [P]      rows of earlier tiles
    int *whist = toff + a.P;                   // [HW][P]
    int *pp = whist + HW * a.P;                // [tile_tokens * k]
    __shared__ int warp_tot[LAYOUT_WARPS + 1];

    pdl_launch_dependents();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int tile = blockIdx.x;
    const int NT = a.n_tiles;
    const int t0 = tile * a.tile_tokens;
    const int nt = min(a.tile_tokens, a.T - t0);
    const int npairs = nt * a.k;
    for (int i = threadIdx.x; i < HW * a.P; i += blockDim.x) whist[i] = 0;
    pdl_wait();

    if (FUSED) {
        // per expert: rows in tiles before this one, and in all tiles.  Four
        // consecutive lanes share a column, each summing every fourth tile
        // with four loads in flight, then combine by shuffles.
        // NT <= 64, so a thread's share is at most 16 tiles: all its loads
        // are issued before any is used (one L2 round trip)
        constexpr int PARTS = 4;
        constexpr int PER = LAYOUT_FUSED_MAX_TILES / PARTS;
        for (int base = 0; base < a.P; base += LAYOUT_THREADS / PARTS) {
            const int p = base + (int)threadIdx.x / PARTS;
            const int part = threadIdx.x % PARTS;
            int before = 0, total = 0;
            if (p < a.P) {
                int c[PER];
#pragma unroll
                for (int u = 0; u < PER; ++u) {
                    const int i = part + u * PARTS;
                    c[u] = (i < NT) ? __ldg(a.tile_cnt + (size_t)i * a.P + p) : 0;
                }
#pragma unroll
                for (int u = 0; u < PER; ++u) {
                    before += (part + u * PARTS < tile) ? c[u] : 0;
                    total += c[u];
                }
            }
#pragma unroll
            for (int off = 1; off < PARTS; off <<= 1) {
                before += __shfl_xor_sync(FULL_MASK, before, off);
                total += __shfl_xor_sync(FULL_MASK, total, off);
            }
            if (part == 0 && p < a.P) {
                toff[p] = before;
                eoff[p] = total;
            }
        }
    } else {
        for (int p = threadIdx.x; p < a.P; p += blockDim.x) {
            toff[p] = a.tile_cnt[(size_t)tile * a.P + p];  // exclusive, from the scan
            eoff[p] = a.cnt_expert[p];
        }
    }
    int bad = 0;  // reported below from the count kernel's tile status words
    for (int i = threadIdx.x; i < npairs; i += blockDim.x)
        pp[i] = phys_expert(a, t0 + i / a.k, i % a.k, bad);
    __syncthreads();

    if (tile == 0) {
        if (FUSED) {
            for (int p = threadIdx.x; p < a.P; p += blockDim.x) a.cnt_expert[p] = eoff[p];
            // one warp per rank, lanes over tiles (NT <= 64: two loads each)
            for (int r = warp; r < a.R; r += LAYOUT_WARPS) {
                int sum = 0;
                for (int i = lane; i < NT; i += 32) sum += __ldg(a.tile_tok + (size_t)i * a.R + r);
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(FULL_MASK, sum, off);
                if (lane == 0) a.tok_rank[r] = sum;
            }
        }
        if (a.dev_status != nullptr && threadIdx.x < 32) {
            int st = 0;
            for (int i = threadIdx.x; i < NT; i += 32) st |= a.tile_bad[i];
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) st |= __shfl_xor_sync(FULL_MASK, st, off);
            if (threadIdx.x == 0) *a.dev_status = st;
        }
    }
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

    // warps w < HW each own a contiguous share of the tile's pairs, in (t, j)
    // order (warps w >= HW get an empty share)
    const int per = (npairs + HW - 1) / HW;
    const int lo = warp < HW ? min(npairs, warp * per) : npairs;
    const int hi = warp < HW ? min(npairs, lo + per) : npairs;
    int *my = whist + (warp < HW ? warp : 0) * a.P;
    for (int i = lo + lane; i < hi; i += 32) {
        const int p = pp[i];
        if (p >= 0) atomicAdd(&my[p], 1);
    }
    __syncthreads();
    // per expert: first row of each share = expert start + rows of earlier
    // tiles + rows of earlier shares in this tile
    for (int p = threadIdx.x; p < a.P; p += blockDim.x) {
        int base = eoff[p] + toff[p];
        for (int w = 0; w < HW; ++w) {
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
    if (bytes > 48 * 1024)
        cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

}  // namespace

cudaError_t launch_layout(const LayoutArgs &a, cudaStream_t s)
{
    cudaError_t err;
    if (a.T == 0) return launch_pdl(layout_empty_kernel, dim3(1), dim3(256), 0, s, a);
    const int NT = a.n_tiles;
    const size_t pairs = (size_t)a.tile_tokens * a.k;
    const size_t sm_count = sizeof(int) * ((size_t)a.P + a.R + pairs);
    const size_t sm_slot =
        sizeof(int) * ((size_t)2 * a.P + 1 + (size_t)a.hist_warps * a.P + pairs);
    const bool fused = NT <= LAYOUT_FUSED_MAX_TILES;
    opt_in_smem((const void *)layout_count_kernel, sm_count);
    opt_in_smem(fused ? (const void *)layout_slot_kernel<true> : (const void *)layout_slot_kernel<false>,
                sm_slot);
    err = launch_pdl(layout_count_kernel, dim3(NT), dim3(LAYOUT_THREADS), sm_count, s, a);
    if (err != cudaSuccess) return err;
    if (fused) return launch_pdl(layout_slot_kernel<true>, dim3(NT), dim3(LAYOUT_THREADS), sm_slot, s, a);
    const int cols = a.P + a.R;
    err = launch_pdl(layout_scan_kernel, dim3((cols + SCAN_WARPS - 1) / SCAN_WARPS),
                     dim3(SCAN_THREADS), 0, s, a);
    if (err != cudaSuccess) return err;
    return launch_pdl(layout_slot_kernel<false>, dim3(NT), dim3(LAYOUT_THREADS), sm_slot, s, a);
}

}  // namespace ep
