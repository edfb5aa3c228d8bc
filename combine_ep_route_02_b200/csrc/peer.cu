// Expert parallelism over peer memory: the dispatch and combine all-to-alls
// as stores into, and loads from, the other ranks' buffers, with no
// collective library in between.
//
// Dispatch and combine are the two all-to-alls around the experts
// (Perplexity blog, section "Expert Parallelism"); on NVLink / NVSwitch every
// GPU can store to and load from every peer's memory directly, so the
// quantised rows are written once, straight into the receive buffer of the
// rank that owns their expert, and the combine gathers the expert outputs
// straight from the ranks that hold them.
//
// Ranks and tables.  W ranks; a process serves ranks rank0 .. rank0+n_local-1
// on its GPU (one rank per GPU, or several logical ranks on one GPU).  Rank q
// owns physical experts [q*epr, (q+1)*epr), epr = P/W.  Every rank-indexed
// table (receive rows, scales, expert outputs, count board, control words) is
// a device array of W device pointers as this process sees them.
//
// Receive order at rank q: by local expert e, then by source rank s, then in
// the source's own (token, j) order; each expert's block starts on a multiple
// of row_align.  A source therefore needs every rank's per-expert counts: the
// counts are all-gathered first (ep_peer_counts), and each source computes
// where its rows go at every destination.
//
// Control words of a rank (int32 [8], zeroed once when allocated, persistent
// across steps):
//   [0] count messages received   (+1 per source per step)
//   [1] data messages received    (+1 per source per step, after its rows)
//   [2] expert outputs ready: the step number, set by the rank itself
//   [3] step number of this rank  (its own counter, +1 per ep_peer_counts)
//   [4] dispatch blocks finished  (this rank's own blocks; reset each step)
//   [5] error bits of the last wait that gave up
// Every rank makes the same calls in the same order, so step numbers agree.
// Each wait is bounded and reports EP_DEV_TIMEOUT instead of hanging.  No
// load or store here uses TMA, and nothing uses multicast.
#include "../../include/ep.h"
#include "ep_device.cuh"
#include "ep_internal.h"
#include "layout_impl.cuh"
#include "quant.cuh"

namespace ep {

namespace {

constexpr int PEER_THREADS = 256;
constexpr int PEER_TIMEOUT = 4;   // EP_DEV_TIMEOUT
constexpr int PEER_OVERFLOW = 8;  // EP_DEV_OVERFLOW

EP_DEV int ld_acquire_sys(const int32_t *p)
{
    int v;
    asm volatile("ld.acquire.sys.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

EP_DEV void red_release_sys(int32_t *p, int v)
{
    asm volatile("red.release.sys.global.add.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

EP_DEV void st_release_sys(int32_t *p, int v)
{
    asm volatile("st.release.sys.global.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// polls *p until it reaches target; false after `limit` polls
EP_DEV bool wait_at_least(const int32_t *p, int target, uint32_t limit)
{
    for (uint32_t i = 0; i < limit; ++i) {
        if (ld_acquire_sys(p) - target >= 0) return true;
        __nanosleep(64);
    }
    return false;
}

EP_DEV void report(const ep_peer_rank &r, int bits)
{
    if (r.dev_status != nullptr) atomicOr(r.dev_status, bits);
}

// destination rank and row of pair (t, j) of a local rank, from its local
// receive row (the layout's slot): expert p holds local rows
// [expert_off[p], expert_off[p+1]); -1 rank when the pair is invalid
EP_DEV void pair_dest(const int *eoff, const int *doff, int P, int epr, int s_loc, int &q,
                      int &row)
{
    q = -1;
    row = 0;
    if (s_loc < 0 || s_loc >= eoff[P]) return;
    int lo = 0, hi = P;  // eoff[lo] <= s_loc < eoff[hi]
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (eoff[mid] <= s_loc) lo = mid;
        else hi = mid;
    }
    if (doff[lo] < 0) return;  // the counts step gave up
    q = lo / epr;
    row = doff[lo] + (s_loc - eoff[lo]);
}

// 1. all-gather of the per-expert counts, then this rank's destination
//    offsets and receive counts.  One block per local rank.
__global__ void __launch_bounds__(PEER_THREADS)
peer_counts_kernel(ep_peer_group g, const ep_peer_rank *ranks, uint32_t limit)
{
    extern __shared__ int sm[];
    __shared__ int warp_tot[PEER_THREADS / 32 + 1];
    __shared__ int step_sh, ok_sh;
    const int W = g.world, P = g.P, epr = P / W, A = g.row_align;
    const int l = blockIdx.x, me = g.rank0 + l, tid = threadIdx.x;
    const ep_peer_rank &r = ranks[l];
    int *tot = sm;            // [P] padded totals over all sources, then their scan
    int *pre = sm + P;        // [P] rows of sources before this one
    int32_t *my_flags = g.flags[me];

    pdl_launch_dependents();
    pdl_wait();
    if (tid == 0) {
        step_sh = my_flags[3] + 1;  // only this rank writes its step number
        my_flags[3] = step_sh;
    }
    // this rank's counts into row `me` of every rank's board
    for (int q = 0; q < W; ++q)
        for (int p = tid; p < P; p += PEER_THREADS) g.board[q][(size_t)me * P + p] = r.cnt_expert[p];
    __syncthreads();
    if (tid == 0) {
        __threadfence_system();  // cumulative over the block's board stores
        for (int q = 0; q < W; ++q) red_release_sys(&g.flags[q][0], 1);
        ok_sh = wait_at_least(&my_flags[0], W * step_sh, limit);
        if (!ok_sh) my_flags[5] |= PEER_TIMEOUT;
    }
    __syncthreads();
    if (!ok_sh) {
        // no destination rows: the dispatch and combine skip every pair
        for (int p = tid; p < P; p += PEER_THREADS) r.dest_off[p] = -1;
        if (tid == 0) {
            *r.recv_rows = 0;
            report(r, PEER_TIMEOUT);
        }
        return;
    }
    const int32_t *board = g.board[me];  // [W][P], every source's counts
    for (int p = tid; p < P; p += PEER_THREADS) {
        int t = 0, b = 0;
        for (int s = 0; s < W; ++s) {
            const int c = __ldcg(board + (size_t)s * P + p);
            t += c;
            b += s < me ? c : 0;
        }
        tot[p] = (t + A - 1) / A * A;
        pre[p] = b;
        if (p >= me * epr && p < (me + 1) * epr)
            for (int s = 0; s < W; ++s)
                r.recv_cnt[(size_t)(p - me * epr) * W + s] = __ldcg(board + (size_t)s * P + p);
    }
    __syncthreads();
    // destination row of this rank's first pair of expert p: the padded
    // rows of the destination's earlier experts, then earlier sources' rows
    const int total = layout_impl::block_exclusive_scan<PEER_THREADS>(tot, P, warp_tot);
    for (int p = tid; p < P; p += PEER_THREADS) {
        const int q = p / epr;
        r.dest_off[p] = tot[p] - tot[q * epr] + pre[p];
    }
    if (tid == 0) {
        const int end = me + 1 < W ? tot[(me + 1) * epr] : total;
        *r.recv_rows = end - tot[me * epr];
    }
}

// 1b. every pair's destination rank and row, for the dispatch and combine.
//     Grid: n_local x bpr blocks, a thread per pair.
__global__ void __launch_bounds__(PEER_THREADS)
peer_pairs_kernel(ep_peer_group g, const ep_peer_rank *ranks, int k, int bpr)
{
    extern __shared__ int sm[];
    const int P = g.P, epr = P / g.world;
    const int l = blockIdx.x / bpr, part = blockIdx.x % bpr, tid = threadIdx.x;
    const ep_peer_rank &r = ranks[l];
    int *eoff = sm;           // [P + 1] this rank's local expert offsets
    int *doff = sm + P + 1;   // [P] destination offsets
    pdl_launch_dependents();
    pdl_wait();
    for (int p = tid; p <= P; p += PEER_THREADS) eoff[p] = r.expert_off[p];
    for (int p = tid; p < P; p += PEER_THREADS) doff[p] = r.dest_off[p];
    __syncthreads();
    int overflow = 0;
    for (int i = part * PEER_THREADS + tid; i < r.T * k; i += bpr * PEER_THREADS) {
        int q, row;
        pair_dest(eoff, doff, P, epr, r.slot[i], q, row);
        if (q >= 0 && row >= g.cap) {
            overflow = PEER_OVERFLOW;
            q = -1;
        }
        reinterpret_cast<int2 *>(r.pair_dest)[i] = make_int2(q, row);
    }
    if (overflow) report(r, overflow);
}

// 2. dispatch: each token's row quantised once (1x128 e4m3) and stored k
//    times into the owning ranks' receive buffers; the last block of a rank
//    tells every destination that this source's rows are complete.
//    Grid: n_local x bpr blocks; within a rank, a thread owns a 16-element
//    chunk of a row at a time (the flat walk of the local dispatch), and the
//    8 lanes of a 128-element block reduce its amax together.
__global__ void __launch_bounds__(PEER_THREADS)
peer_dispatch_kernel(ep_peer_group g, const ep_peer_rank *ranks, int H, int k, int bpr)
{
    extern __shared__ __align__(16) unsigned char psm[];
    __shared__ int last_sh;
    const int W = g.world;
    const int l = blockIdx.x / bpr, part = blockIdx.x % bpr, me = g.rank0 + l;
    const int tid = threadIdx.x;
    const ep_peer_rank &r = ranks[l];
    // the ranks' receive rows and scales, as this process addresses them
    uint8_t **rx = reinterpret_cast<uint8_t **>(psm);
    float **rs = reinterpret_cast<float **>(psm) + W;
    for (int q = tid; q < W; q += PEER_THREADS) {
        rx[q] = static_cast<uint8_t *>(g.recv_x[q]);
        rs[q] = g.recv_scale[q];
    }
    __syncthreads();
    pdl_launch_dependents();
    pdl_wait();
    const int2 *pd = reinterpret_cast<const int2 *>(r.pair_dest);
    const int S = H >> 7, cpr = H >> 4;  // cpr is a multiple of 8
    const uint16_t *x = static_cast<const uint16_t *>(r.x);
    const long long total = (long long)r.T * cpr;
    const long long stride = (long long)bpr * PEER_THREADS;
    ChunkWalk it((long long)part * PEER_THREADS + tid, stride, cpr);
    // block-uniform bound: every lane reaches the shuffles; total and the
    // stride are multiples of 8, so a lane octet is all active or all idle
    for (long long base = (long long)part * PEER_THREADS; base < total; base += stride, it.next()) {
        const bool active = it.t < r.T;
        const int t = it.t, c = it.c;
        uint4 lo = make_uint4(0, 0, 0, 0), hi = make_uint4(0, 0, 0, 0);
        if (active) {
            lo = ld_stream(x + (size_t)t * H + (size_t)c * 16);
            hi = ld_stream(x + (size_t)t * H + (size_t)c * 16 + 8);
        }
        float scale;
        const uint4 qv = quant::quant_chunk(lo, hi, scale);
        if (active)
            for (int j = 0; j < k; ++j) {
                const int2 qr = pd[(size_t)t * k + j];
                if (qr.x < 0) continue;
                const size_t row = (size_t)qr.y;
                *reinterpret_cast<uint4 *>(rx[qr.x] + row * H + (size_t)c * 16) = qv;
                if ((c & 7) == 0) rs[qr.x][row * S + (c >> 3)] = scale;
            }
    }
    // this block's rows are visible everywhere before it counts itself
    // done: the block's barrier orders its threads' stores before thread 0's
    // system-scope fence, which is cumulative over them
    __syncthreads();
    if (tid == 0) {
        __threadfence_system();
        const int done = atomicAdd(&g.flags[me][4], 1);
        last_sh = done == bpr - 1;
    }
    __syncthreads();
    if (last_sh && tid == 0) {
        __threadfence_system();
        g.flags[me][4] = 0;
        for (int q = 0; q < W; ++q) red_release_sys(&g.flags[q][1], 1);
    }
}

// 3. a rank waits for every source's rows (before its experts run).  One
//    block per local rank.
__global__ void peer_wait_kernel(ep_peer_group g, const ep_peer_rank *ranks, uint32_t limit)
{
    pdl_launch_dependents();
    pdl_wait();
    const int me = g.rank0 + blockIdx.x;
    if (threadIdx.x == 0) {
        int32_t *f = g.flags[me];
        if (!wait_at_least(&f[1], g.world * f[3], limit)) {
            f[5] |= PEER_TIMEOUT;
            report(ranks[blockIdx.x], PEER_TIMEOUT);
        }
    }
}

// 4. a rank's expert outputs are ready for the sources to read
__global__ void peer_ready_kernel(ep_peer_group g)
{
    pdl_launch_dependents();
    pdl_wait();
    const int me = g.rank0 + blockIdx.x;
    if (threadIdx.x == 0) {
        __threadfence_system();
        st_release_sys(&g.flags[me][2], g.flags[me][3]);
    }
}

// 5. combine: once every rank holding this rank's pairs has its outputs
//    ready, each token's k rows are read from those ranks and summed in j
//    order with the weights, in fp32, rounded once to bf16 (as ep_combine).
//    Grid: n_local x bpr blocks; a thread owns an 8-element chunk of an
//    output row and issues up to 8 row loads before it accumulates.
__global__ void __launch_bounds__(PEER_THREADS)
peer_combine_kernel(ep_peer_group g, const ep_peer_rank *ranks, int H, int k, int bpr,
                    uint32_t limit)
{
    extern __shared__ __align__(16) unsigned char psm[];
    __shared__ int ok_sh;
    const int W = g.world;
    const int l = blockIdx.x / bpr, part = blockIdx.x % bpr, me = g.rank0 + l;
    const int tid = threadIdx.x;
    const ep_peer_rank &r = ranks[l];
    const uint16_t **ys = reinterpret_cast<const uint16_t **>(psm);  // [W]
    for (int q = tid; q < W; q += PEER_THREADS) ys[q] = static_cast<const uint16_t *>(g.y[q]);
    pdl_launch_dependents();
    pdl_wait();
    if (tid == 0) {
        const int step = g.flags[me][3];
        bool ok = true;
        for (int q = 0; q < W && ok; ++q) ok = wait_at_least(&g.flags[q][2], step, limit);
        ok_sh = ok;
        if (!ok) report(r, PEER_TIMEOUT);
    }
    __syncthreads();
    if (!ok_sh) return;
    constexpr int BATCH = 8;
    const int cpr = H >> 3;
    const int2 *pd = reinterpret_cast<const int2 *>(r.pair_dest);
    uint16_t *out = static_cast<uint16_t *>(r.out);
    const long long total = (long long)r.T * cpr;
    const long long g0 = (long long)part * PEER_THREADS + tid;
    if (g0 >= total) return;
    for (ChunkWalk it(g0, (long long)bpr * PEER_THREADS, cpr); it.t < r.T; it.next()) {
        const int t = it.t, c = it.c;
        float acc[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] = 0.0f;
        for (int j0 = 0; j0 < k; j0 += BATCH) {
            uint4 v[BATCH];
            float wj[BATCH];
            bool ok[BATCH];
#pragma unroll
            for (int u = 0; u < BATCH; ++u) {
                const int j = j0 + u;
                const int2 qr = j < k ? pd[(size_t)t * k + j] : make_int2(-1, 0);
                ok[u] = qr.x >= 0;
                wj[u] = ok[u] ? __ldg(r.topk_w + (size_t)t * k + j) : 0.0f;
                v[u] = ok[u] ? ld_stream(ys[qr.x] + (size_t)qr.y * H + (size_t)c * 8)
                             : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int u = 0; u < BATCH; ++u) {
                if (!ok[u]) continue;
                const uint32_t pk[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
                for (int m = 0; m < 4; ++m) {
                    acc[2 * m] = __fadd_rn(acc[2 * m], __fmul_rn(wj[u], bf16_lo(pk[m])));
                    acc[2 * m + 1] = __fadd_rn(acc[2 * m + 1], __fmul_rn(wj[u], bf16_hi(pk[m])));
                }
            }
        }
        uint4 o;
        o.x = pack_bf16x2(acc[0], acc[1]);
        o.y = pack_bf16x2(acc[2], acc[3]);
        o.z = pack_bf16x2(acc[4], acc[5]);
        o.w = pack_bf16x2(acc[6], acc[7]);
        *reinterpret_cast<uint4 *>(out + (size_t)t * H + (size_t)c * 8) = o;
    }
}

ep_status check_group(const ep_peer_group &g, const ep_peer_rank *ranks, bool need_ranks = true)
{
    if (g.world < 1 || g.world > 1024 || g.n_local < 1 || g.rank0 < 0 ||
        g.rank0 + g.n_local > g.world)
        return EP_ERR_INVALID;
    if (g.P < 1 || g.P % g.world != 0 || g.row_align < 1 || g.cap < 0) return EP_ERR_INVALID;
    if (g.P > MAX_PHYS || g.row_align > MAX_ROW_ALIGN) return EP_ERR_UNSUPPORTED;
    if (!g.board || !g.flags || (need_ranks && !ranks)) return EP_ERR_INVALID;
    // the local ranks' blocks of one launch wait for one another: all resident
    if (g.n_local > device_sm_count()) return EP_ERR_UNSUPPORTED;
    return EP_OK;
}

// blocks per local rank: the GPU's resident blocks shared out over the local
// ranks, and no more than the largest rank's chunks need
int peer_blocks_per_rank(int n_local, int max_T, int chunks_per_row)
{
    int b = (device_sm_count() * 8 + n_local - 1) / n_local;
    const long long need = ((long long)max_T * chunks_per_row + PEER_THREADS - 1) / PEER_THREADS;
    if (need < b) b = (int)need;
    return b < 1 ? 1 : b;
}

}  // namespace
}  // namespace ep

using namespace ep;

extern "C" {

ep_status ep_peer_counts(ep_peer_group g, const ep_peer_rank *ranks, int k, int max_T,
                         ep_stream_t stream)
{
    EP_TRACE("ep_peer_counts");
    const ep_status st = check_group(g, ranks);
    if (st != EP_OK) return st;
    if (k < 1 || max_T < 0) return EP_ERR_INVALID;
    if (k > MAX_TOPK) return EP_ERR_UNSUPPORTED;
    const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const size_t smem = sizeof(int) * 2 * (size_t)g.P;
    if (smem > 48 * 1024)
        cudaFuncSetAttribute(peer_counts_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
    if (launch_pdl(peer_counts_kernel, dim3(g.n_local), dim3(PEER_THREADS), smem, s, g, ranks,
                   wait_limit()) != cudaSuccess)
        return EP_ERR_CUDA;
    // the pairs' destinations: a thread per pair of the largest rank
    int bpr = (int)(((long long)max_T * k + PEER_THREADS - 1) / PEER_THREADS);
    if (bpr < 1) bpr = 1;
    const size_t smem2 = sizeof(int) * (2 * (size_t)g.P + 1);
    if (smem2 > 48 * 1024)
        cudaFuncSetAttribute(peer_pairs_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem2);
    return launch_pdl(peer_pairs_kernel, dim3(g.n_local * bpr), dim3(PEER_THREADS), smem2, s, g,
                      ranks, k, bpr) == cudaSuccess
               ? EP_OK
               : EP_ERR_CUDA;
}

ep_status ep_peer_dispatch(ep_peer_group g, const ep_peer_rank *ranks, int H, int k,
                           int max_T, ep_stream_t stream)
{
    EP_TRACE("ep_peer_dispatch");
    ep_status st = check_group(g, ranks);
    if (st != EP_OK) return st;
    if (H < 128 || H % 128 != 0 || k < 1 || max_T < 0) return EP_ERR_INVALID;
    if (k > MAX_TOPK) return EP_ERR_UNSUPPORTED;
    if (!g.recv_x || !g.recv_scale) return EP_ERR_INVALID;
    const int bpr = peer_blocks_per_rank(g.n_local, max_T, H / 16);
    const size_t smem = 2 * sizeof(void *) * (size_t)g.world;
    if (smem > 48 * 1024)
        cudaFuncSetAttribute(peer_dispatch_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
    return launch_pdl(peer_dispatch_kernel, dim3(g.n_local * bpr), dim3(PEER_THREADS), smem,
                      reinterpret_cast<cudaStream_t>(stream), g, ranks, H, k, bpr) == cudaSuccess
               ? EP_OK
               : EP_ERR_CUDA;
}

ep_status ep_peer_wait_dispatch(ep_peer_group g, const ep_peer_rank *ranks, ep_stream_t stream)
{
    EP_TRACE("ep_peer_wait_dispatch");
    const ep_status st = check_group(g, ranks);
    if (st != EP_OK) return st;
    return launch_pdl(peer_wait_kernel, dim3(g.n_local), dim3(32), 0,
                      reinterpret_cast<cudaStream_t>(stream), g, ranks, wait_limit()) == cudaSuccess
               ? EP_OK
               : EP_ERR_CUDA;
}

ep_status ep_peer_experts_ready(ep_peer_group g, ep_stream_t stream)
{
    EP_TRACE("ep_peer_experts_ready");
    const ep_status st = check_group(g, nullptr, false);
    if (st != EP_OK) return st;
    return launch_pdl(peer_ready_kernel, dim3(g.n_local), dim3(32), 0,
                      reinterpret_cast<cudaStream_t>(stream), g) == cudaSuccess
               ? EP_OK
               : EP_ERR_CUDA;
}

ep_status ep_peer_combine(ep_peer_group g, const ep_peer_rank *ranks, int H, int k, int max_T,
                          ep_stream_t stream)
{
    EP_TRACE("ep_peer_combine");
    ep_status st = check_group(g, ranks);
    if (st != EP_OK) return st;
    if (H < 8 || H % 8 != 0 || k < 1 || max_T < 0) return EP_ERR_INVALID;
    if (k > MAX_TOPK) return EP_ERR_UNSUPPORTED;
    if (!g.y) return EP_ERR_INVALID;
    const int bpr = peer_blocks_per_rank(g.n_local, max_T, H / 8);
    const size_t smem = sizeof(void *) * (size_t)g.world;
    return launch_pdl(peer_combine_kernel, dim3(g.n_local * bpr), dim3(PEER_THREADS), smem,
                      reinterpret_cast<cudaStream_t>(stream), g, ranks, H, k, bpr,
                      wait_limit()) == cudaSuccess
               ? EP_OK
               : EP_ERR_CUDA;
}

}  // extern "C"
