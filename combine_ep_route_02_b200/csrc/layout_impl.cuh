// Dispatch layout, device side: counting and ordering one tile of tokens.
// Included by the layout kernels and by the fused small-batch kernel.
#pragma once

#include "ep_device.cuh"
#include "ep_internal.h"

namespace ep {
namespace layout_impl {


constexpr int BAD_EXPERT = 1;
constexpr int BAD_REPLICA = 2;

// physical expert of logical expert e for token t; -1 (and a status bit)
// when invalid
EP_DEV int phys_of_id(const LayoutArgs &a, int t, int e, int &bad)
{
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

// Fills pp[0..npairs) with the physical experts of the tile's pairs (and
// counts them in hist when given).  Each thread issues the loads of up to
// eight of its pairs before using any, so a tile costs few L2 round trips.
EP_DEV void fill_pairs(const LayoutArgs &a, int t0, int npairs, int *pp, int *hist, int &bad)
{
    constexpr int U = 8;
    const int32_t *ids = a.topk_idx + (size_t)t0 * a.k;
    for (int i0 = threadIdx.x; i0 < npairs; i0 += U * blockDim.x) {
        int e[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int i = i0 + u * (int)blockDim.x;
            e[u] = (i < npairs) ? ids[i] : 0;
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int i = i0 + u * (int)blockDim.x;
            if (i < npairs) {
                // the token index only matters for the replica choice
                const int t = a.phys_of != nullptr ? t0 + i / a.k : 0;
                const int p = phys_of_id(a, t, e[u], bad);
                pp[i] = p;
                if (hist != nullptr && p >= 0) atomicAdd(&hist[p], 1);
            }
        }
    }
}

// floor(n / d) for 0 <= n < 2^22 and 1 <= d <= 2^22 without an integer
// division: (n + 1/2) / d lies at least 1/(2d) from the nearest integer, far
// more than the rounding error of the fp32 product, so truncation is exact.
EP_DEV int small_div(int n, float inv_d)
{
    return __float2int_rz(__fmul_rn((float)n + 0.5f, inv_d));
}

// Shared memory of count_tile, in ints: hist [P], tokr [R], pairs
// [tile_tokens * k], then (8-byte aligned) the token rank masks [tile_tokens]
// as 64-bit words.
inline size_t count_smem_ints(int P, int R, int tile_tokens, int k)
{
    return (((size_t)P + R + (size_t)tile_tokens * k + 1) & ~(size_t)1) + 2 * (size_t)tile_tokens;
}

// Counts one tile (the block's threads cooperate; smem: count_smem_ints
// ints; bad_sh: one shared int).  Writes tile_cnt / tile_tok / tile_bad row
// `tile` and in_rank for the tile's tokens; hist and tokr stay in shared
// memory for a caller that lays the tile out in the same block.
EP_DEV void count_tile(const LayoutArgs &a, int tile, int *smem, int *bad_sh_p)
{
    int *hist = smem;          // [P]
    int *tokr = hist + a.P;    // [R]
    int *pp = tokr + a.R;      // [tile_tokens * k]
    unsigned long long *tmask = reinterpret_cast<unsigned long long *>(
        smem + (((size_t)a.P + a.R + (size_t)a.tile_tokens * a.k + 1) & ~(size_t)1));
    int &bad_sh = *bad_sh_p;
    const int t0 = tile * a.tile_tokens;
    const int nt = min(a.tile_tokens, a.T - t0);
    const int npairs = nt * a.k;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;

    for (int i = threadIdx.x; i < a.P; i += blockDim.x) hist[i] = 0;
    for (int i = threadIdx.x; i < a.R; i += blockDim.x) tokr[i] = 0;
    if (threadIdx.x == 0) bad_sh = 0;
    __syncthreads();

    int bad = 0;
    fill_pairs(a, t0, npairs, pp, hist, bad);
    if (bad) atomicOr(&bad_sh, bad);
    __syncthreads();

    const int epr = a.P / a.R;
    const float inv_epr = 1.0f / (float)epr, inv_R = 1.0f / (float)a.R;
    if (a.R <= 64) {
        // the set of ranks each token reaches, as a bit mask
        for (int tl = threadIdx.x; tl < nt; tl += blockDim.x) {
            unsigned long long m = 0;
            for (int j = 0; j < a.k; ++j) {
                const int p = pp[tl * a.k + j];
                if (p >= 0) m |= 1ull << small_div(p, inv_epr);
            }
            tmask[tl] = m;
        }
        __syncthreads();
        // tokens per rank: a ballot per rank over each warp's 32 tokens,
        // one shared atomic per (warp, rank)
        int c_lo = 0, c_hi = 0;  // counts of ranks lane and lane + 32
        for (int base = warp * 32; base < nt; base += nwarps * 32) {  // warp-uniform
            const unsigned long long m = base + lane < nt ? tmask[base + lane] : 0ull;
            for (int r = 0; r < a.R; ++r) {
                const int c = __popc(__ballot_sync(FULL_MASK, (m >> r) & 1ull));
                if (r < 32) c_lo += (lane == r) ? c : 0;
                else c_hi += (lane == r - 32) ? c : 0;
            }
        }
        if (lane < a.R && c_lo) atomicAdd(&tokr[lane], c_lo);
        if (lane + 32 < a.R && c_hi) atomicAdd(&tokr[lane + 32], c_hi);
        // in_rank rows: the tile's rows are one contiguous byte range;
        // consecutive threads write consecutive 4-byte words of it
        uint8_t *dst = a.in_rank + (size_t)t0 * a.R;
        const int nbytes = nt * a.R;
        const bool words = (reinterpret_cast<uintptr_t>(dst) & 3) == 0;
        const int nw = words ? nbytes >> 2 : 0;
        for (int w = threadIdx.x; w < nw; w += blockDim.x) {
            int tl = small_div(4 * w, inv_R), r = 4 * w - tl * a.R;
            uint32_t v = 0;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                v |= (uint32_t)((tmask[tl] >> r) & 1ull) << (8 * q);
                if (++r == a.R) {
                    r = 0;
                    ++tl;
                }
            }
            reinterpret_cast<uint32_t *>(dst)[w] = v;
        }
        for (int b = 4 * nw + threadIdx.x; b < nbytes; b += blockDim.x) {
            const int tl = small_div(b, inv_R), r = b - tl * a.R;
            dst[b] = (uint8_t)((tmask[tl] >> r) & 1ull);
        }
    } else {
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
    }
    __syncthreads();

    for (int i = threadIdx.x; i < a.P; i += blockDim.x) a.tile_cnt[(size_t)tile * a.P + i] = hist[i];
    for (int i = threadIdx.x; i < a.R; i += blockDim.x) a.tile_tok[(size_t)tile * a.R + i] = tokr[i];
    if (threadIdx.x == 0) a.tile_bad[tile] = bad_sh;
}

// exclusive scan of n ints held in shared memory (n <= MAX_PHYS), in place;
// returns the total.  Every thread of the block must call it.
template <int NTHREADS>
EP_DEV int block_exclusive_scan(int *v, int n, int *warp_tot)
{
    constexpr int NWARPS = NTHREADS / 32;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int per = (n + NTHREADS - 1) / NTHREADS;
    const int lo = min(n, threadIdx.x * per), hi = min(n, lo + per);
    int local = 0;
    for (int i = lo; i < hi; ++i) local += v[i];
    const int incl = warp_inclusive_scan(local);
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const int wt = (lane < NWARPS) ? warp_tot[lane] : 0;
        const int wincl = warp_inclusive_scan(wt);
        if (lane < NWARPS) warp_tot[lane] = wincl - wt;
        if (lane == NWARPS - 1) warp_tot[NWARPS] = wincl;
    }
    __syncthreads();
    int run = warp_tot[warp] + incl - local;
    for (int i = lo; i < hi; ++i) {
        const int c = v[i];
        v[i] = run;
        run += c;
    }
    const int total = warp_tot[NWARPS];
    __syncthreads();
    return total;
}

// Orders one tile's pairs into receive rows (smem: 2P + 1 + hist_warps*P +
// tile_tokens*k ints; warp_tot: NTHREADS/32 + 1 shared ints).  Tile 0 also
// writes the batch-wide outputs.  FUSED: the tile histograms are raw counts
// and are summed here; otherwise tile_cnt already holds exclusive per-tile
// offsets and cnt_expert the totals.  ready (single-tile batches counted by
// the same block, in shared memory): the pairs' physical experts [npairs],
// then the expert counts [P], the rank token counts [R] and the status bits.
template <int NTHREADS, bool FUSED>
EP_DEV void slot_tile(const LayoutArgs &a, int tile, int *smem, int *warp_tot,
                      const int *ready = nullptr)
{
    constexpr int NWARPS = NTHREADS / 32;
    const int HW = a.hist_warps;
    int *eoff = smem;                          // [P + 1]  expert start rows
    int *toff = eoff + a.P + 1;                // [P]      rows of earlier tiles
    int *whist = toff + a.P;                   // [HW][P]
    int *pp = whist + HW * a.P;                // [tile_tokens * k]

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int NT = a.n_tiles;
    const int t0 = tile * a.tile_tokens;
    const int nt = min(a.tile_tokens, a.T - t0);
    const int npairs = nt * a.k;
    for (int i = threadIdx.x; i < HW * a.P; i += blockDim.x) whist[i] = 0;

    const int *ready_hist = ready != nullptr ? ready + npairs : nullptr;
    if (FUSED && ready != nullptr) {
        for (int p = threadIdx.x; p < a.P; p += blockDim.x) {
            toff[p] = 0;
            eoff[p] = ready_hist[p];
        }
    } else if (FUSED) {
        // per expert: rows in tiles before this one, and in all tiles.  Four
        // consecutive lanes share a column, each summing every fourth tile
        // with four loads in flight, then combine by shuffles.
        // NT <= 64, so a thread's share is at most 16 tiles: all its loads
        // are issued before any is used (one L2 round trip)
        constexpr int PARTS = 4;
        constexpr int PER = LAYOUT_FUSED_MAX_TILES / PARTS;
        for (int base = 0; base < a.P; base += NTHREADS / PARTS) {
            const int p = base + (int)threadIdx.x / PARTS;
            const int part = threadIdx.x % PARTS;
            int before = 0, total = 0;
            if (p < a.P) {
                int c[PER];
#pragma unroll
                for (int u = 0; u < PER; ++u) {
                    const int i = part + u * PARTS;
                    c[u] = (i < NT) ? a.tile_cnt[(size_t)i * a.P + p] : 0;
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
    if (ready != nullptr) {  // the same block counted this tile already
        for (int i = threadIdx.x; i < npairs; i += blockDim.x) pp[i] = ready[i];
    } else {
        fill_pairs(a, t0, npairs, pp, nullptr, bad);
    }
    __syncthreads();

    if (tile == 0) {
        if (FUSED && ready != nullptr) {
            for (int p = threadIdx.x; p < a.P; p += blockDim.x) a.cnt_expert[p] = eoff[p];
            for (int r = threadIdx.x; r < a.R; r += blockDim.x) a.tok_rank[r] = ready_hist[a.P + r];
        } else if (FUSED) {
            for (int p = threadIdx.x; p < a.P; p += blockDim.x) a.cnt_expert[p] = eoff[p];
            // one warp per rank, lanes over tiles (NT <= 64: two loads each)
            for (int r = warp; r < a.R; r += NWARPS) {
                int sum = 0;
                for (int i = lane; i < NT; i += 32) sum += a.tile_tok[(size_t)i * a.R + r];
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(FULL_MASK, sum, off);
                if (lane == 0) a.tok_rank[r] = sum;
            }
        }
        if (a.dev_status != nullptr && ready != nullptr) {
            if (threadIdx.x == 0) *a.dev_status = ready_hist[a.P + a.R];
        } else if (a.dev_status != nullptr && threadIdx.x < 32) {
            int st = 0;
            for (int i = threadIdx.x; i < NT; i += 32) st |= a.tile_bad[i];
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) st |= __shfl_xor_sync(FULL_MASK, st, off);
            if (threadIdx.x == 0) *a.dev_status = st;
        }
    }
    if (a.row_align > 1) {
        // GEMM layout: every expert's rows start on a multiple of the row
        // tile (same thread-to-expert mapping as the loops above)
        const int A = a.row_align;
        for (int p = threadIdx.x; p < a.P; p += blockDim.x) eoff[p] = (eoff[p] + A - 1) / A * A;
        __syncthreads();
    }
    const int total = block_exclusive_scan<NTHREADS>(eoff, a.P, warp_tot);
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
        if (a.row_align > 1) {
            // padding rows after each expert's pairs: src = -1 (a warp per
            // expert; cnt_expert was written by this block above, or by the
            // scan kernel)
            for (int p = warp; p < a.P; p += NWARPS) {
                const int first = eoff[p] + a.cnt_expert[p];
                for (int r = first + lane; r < eoff[p + 1]; r += 32) a.src[r] = -1;
            }
        }
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

}  // namespace layout_impl
}  // namespace ep
