// Routing, dispatch layout and dispatch of a small (decode-sized) batch in
// one kernel.
//
// The DeepEP V2 summary (section "Usage for training, prefill and decoding")
// gives decoding its own low-latency path, and the Perplexity blog (section
// "CUDA Graph") runs the small-batch MoE steps from device-side counts under
// CUDA graphs.  For such a batch every separate launch and every global
// round trip between the steps costs more than the bytes do, so here one
// kernel does all three:
//
//   1. each block starts the TMA loads of its own tokens' rows of x, then
//      routes those tokens (a warp per token) and writes their top-k;
//   2. it arrives on a grid-wide counter, quantises its rows from shared
//      memory while the other blocks finish routing, and waits (bounded) for
//      every block to arrive;
//   3. every block then reads all T*k expert ids from L2 and lays out the
//      whole batch itself: the per-expert counts, their padded exclusive
//      scan and the counts of the pairs before its first token give the
//      receive row of each of its own pairs, so no block waits for another a
//      second time; block 0 also writes the batch-wide arrays;
//   4. each block sends its rows to their k receive rows with TMA bulk
//      stores straight from shared memory.
//
// The grid has at most one block per SM (grid <= SM count), so every block
// is resident; the wait still gives up after a bounded number of polls and
// reports EP_DEV_TIMEOUT instead of hanging.  The counters live in the
// caller's workspace: zero before its first use, and the last block to leave
// clears them again (after a timeout too), so no call needs a memset.
#include "layout_impl.cuh"
#include "quant.cuh"
#include "route_impl.cuh"

namespace ep {

namespace {

constexpr int DEC_THREADS = 256;
constexpr int DEC_WARPS = DEC_THREADS / 32;
constexpr int DEV_TIMEOUT_BIT = 4;  // EP_DEV_TIMEOUT

struct DecodeArgs {
    const uint16_t *x;   // bf16 [T, H]
    int H, fp8, n_rows;
    uint8_t *recv_x;     // e4m3 [n_rows, H] or bf16 [n_rows, H] (as bytes)
    float *recv_scale;   // [n_rows, H/128] when fp8
    int tpb;             // tokens per block
    int scale_bulk;      // scale rows go out by bulk stores (16-byte rows, aligned)
    int *ctrl;           // workspace: [0] arrivals, [1] departures, [2] status bits;
                         // zero before the first call, left zero by every call
    uint32_t wait_limit; // polls of each bounded wait
};

// dynamic shared memory, in order: x rows [tpb][2H] bytes; fp8 codes
// [tpb][H] and scales [tpb][H/128] fp32; then ints: hist [P], run [P],
// eoff [P + 1], pp [T*k]
struct DecodeSmem {
    size_t x_off, q_off, sc_off, int_off, total;
};

__host__ __device__ inline DecodeSmem decode_smem(int tpb, int H, int fp8, int P, int T, int k)
{
    DecodeSmem m;
    m.x_off = 0;
    m.q_off = (size_t)tpb * 2 * H;
    m.sc_off = m.q_off + (fp8 ? (size_t)tpb * H : 0);
    m.int_off = m.sc_off + (fp8 ? (size_t)tpb * (H / 128) * 4 : 0);
    m.int_off = (m.int_off + 15) & ~(size_t)15;
    m.total = m.int_off + sizeof(int) * ((size_t)3 * P + 1 + (size_t)T * k);
    return m;
}

EP_DEV uint32_t ld_acquire(const int *p)
{
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Waits (bounded, every lane) for the block's rows of x, then quantises
// them into the code / scale stage with warps qw, qw + nq, ... of the
// calling warps' set.  Returns false (warp-uniform) if the wait gave up.
EP_DEV bool quantise_rows(const DecodeArgs &d, int nt, uint32_t bar, uint32_t xs, uint32_t qs,
                          uint32_t ss, int qw, int nq)
{
    const int lane = threadIdx.x & 31;
    const bool ok = __all_sync(FULL_MASK, mbar_wait(bar, 0, d.wait_limit));
    if (!ok || !d.fp8) return ok;
    const int H = d.H, cpr = H >> 4;  // cpr is a multiple of 8
    const uint32_t row_bytes = 2u * (uint32_t)H;
    for (int tl = 0; tl < nt; ++tl) {
        const uint32_t in = xs + (uint32_t)tl * row_bytes;
        const uint32_t qo = qs + (uint32_t)(tl * H);
        const uint32_t so = ss + (uint32_t)(tl * (H >> 7)) * 4u;
        // warp-uniform bound; chunk c0 + lane with c0 a multiple of 32, so the
        // 8 lanes of a 128-element block are all active or all idle
        for (int c0 = qw * 32; c0 < cpr; c0 += nq * 32) {
            const int c = c0 + lane;
            const bool act = c < cpr;
            uint4 lo = make_uint4(0, 0, 0, 0), hi = make_uint4(0, 0, 0, 0);
            if (act) {
                lo = lds128(in + 32u * c);
                hi = lds128(in + 32u * c + 16u);
            }
            float scale;
            const uint4 q = quant::quant_chunk(lo, hi, scale);
            if (act) {
                sts128(qo + 16u * c, q);
                if ((c & 7) == 0)
                    asm volatile("st.shared.f32 [%0], %1;" ::"r"(so + 4u * (c >> 3)), "f"(scale)
                                 : "memory");
            }
        }
    }
    fence_proxy_async_smem();  // the stage is read by TMA bulk stores later
    return true;
}

template <int EPL>
__global__ void __launch_bounds__(DEC_THREADS)
route_dispatch_small_kernel(RouteArgs r, LayoutArgs a, DecodeArgs d, int vec4)
{
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ double tab[64];
    __shared__ int bad_sh, xfail_sh, go_sh;
    __shared__ __align__(8) uint64_t xbar;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int NB = gridDim.x, b = blockIdx.x;
    const int T = a.T, k = a.k, P = a.P, R = a.R, H = d.H;
    const int t0 = b * d.tpb;
    const int nt = min(d.tpb, T - t0);  // 1..8: the grid is ceil(T / tpb), tpb <= 8
    const DecodeSmem m = decode_smem(d.tpb, H, d.fp8, P, T, k);
    int *hist = reinterpret_cast<int *>(smem + m.int_off);  // [P]
    int *run = hist + P;                                      // [P]
    int *eoff = run + P;                                      // [P + 1]
    int *pp = eoff + P + 1;                                   // [T * k]
    const uint32_t xs = smem_u32(smem + m.x_off);
    const uint32_t qs = smem_u32(smem + m.q_off);
    const uint32_t ss = smem_u32(smem + m.sc_off);
    const uint32_t bar = smem_u32(&xbar);
    const uint32_t row_bytes = 2u * (uint32_t)H;

    if (tid == 0) {
        mbar_init(bar, 1);
        fence_mbar_init();
        xfail_sh = 0;
    }
    route_impl::load_exp_table(tab);
    __syncthreads();
    pdl_launch_dependents();
    pdl_wait();

    // 1. this block's rows of x into shared memory (they do not depend on
    //    the routing); warps 0 .. nt-1 route one token each while the other
    //    warps quantise the rows (a block of 8 tokens routes with every warp
    //    and quantises afterwards)
    if (tid == 0) {
        mbar_arrive_expect_tx(bar, row_bytes * (uint32_t)nt);
        for (int i = 0; i < nt; ++i)
            bulk_load(xs + (uint32_t)i * row_bytes, d.x + (size_t)(t0 + i) * H, row_bytes, bar);
    }
    if (warp < nt)
        route_impl::route_tokens<EPL>(r.logits, r.bias, t0 + warp + 1, r.E, r.G, r.Kg, r.k,
                                      r.scale, r.renorm, vec4, r.topk_idx, r.topk_w, tab,
                                      t0 + warp, DEC_WARPS);
    else if (!quantise_rows(d, nt, bar, xs, qs, ss, warp - nt, DEC_WARPS - nt) && lane == 0)
        xfail_sh = 1;
    __threadfence();  // this block's top-k is visible before it arrives
    __syncthreads();
    int arrival = 0;
    if (tid == 0) arrival = atomicAdd(&d.ctrl[0], 1);
    if (nt == DEC_WARPS) {
        if (!quantise_rows(d, nt, bar, xs, qs, ss, warp, DEC_WARPS) && lane == 0) xfail_sh = 1;
        __syncthreads();
    }
    const bool x_ok = xfail_sh == 0;
    int status = 0;
    if (!x_ok) {
        status |= DEV_TIMEOUT_BIT;
        // the rows still in flight must land before shared memory is reused
        if (tid == 0) mbar_wait(bar, 0, WAIT_LIMIT_DEFAULT);
    }

    // wait until every block has routed its tokens
    if (tid == 0) {
        bool ok = arrival == NB - 1;
        for (uint32_t i = 0; !ok && i < d.wait_limit; ++i) {
            ok = ld_acquire(&d.ctrl[0]) >= (uint32_t)NB;
            if (!ok) __nanosleep(32);
        }
        go_sh = ok ? 1 : 0;
    }
    __syncthreads();
    const bool all_routed = go_sh != 0;

    if (all_routed) {
        // 2. the layout of the whole batch, in every block
        const int npairs = T * k;
        const int before_end = t0 * k;  // pairs of earlier blocks' tokens
        for (int i = tid; i < P; i += DEC_THREADS) {
            hist[i] = 0;
            run[i] = 0;
        }
        if (tid == 0) bad_sh = 0;
        __syncthreads();
        int bad = 0;
        {
            constexpr int U = 8;  // id loads in flight per thread
            for (int i0 = tid; i0 < npairs; i0 += U * DEC_THREADS) {
                int e[U];
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    const int i = i0 + u * DEC_THREADS;
                    // written by other blocks in this kernel: read from L2
                    e[u] = i < npairs ? __ldcg(r.topk_idx + i) : 0;
                }
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    const int i = i0 + u * DEC_THREADS;
                    if (i < npairs) {
                        const int t = a.phys_of != nullptr ? i / k : 0;
                        const int p = layout_impl::phys_of_id(a, t, e[u], bad);
                        pp[i] = p;
                        if (p >= 0) {
                            atomicAdd(&hist[p], 1);
                            if (i < before_end) atomicAdd(&run[p], 1);
                        }
                    }
                }
            }
        }
        if (bad) atomicOr(&bad_sh, bad);
        __syncthreads();
        status |= bad_sh;  // every block finds the same bits
        const int A = a.row_align;
        if (warp == 0) {
            // exclusive scan of the padded counts by one warp (one block
            // barrier instead of several): lane l takes experts
            // [l * per, (l + 1) * per), per <= 32 since P <= 1024
            const int per = (P + 31) >> 5;
            const int lo = min(P, lane * per), hi = min(P, lo + per);
            int local = 0;
            for (int p = lo; p < hi; ++p) local += (hist[p] + A - 1) / A * A;
            const int incl = warp_inclusive_scan(local);
            int acc = incl - local;
            for (int p = lo; p < hi; ++p) {
                const int c = (hist[p] + A - 1) / A * A;
                eoff[p] = acc;
                run[p] += acc;  // the block's first row of expert p
                acc += c;
            }
            if (lane == 31) eoff[P] = incl;
        }
        __syncthreads();
        const int total = eoff[P];

        const int epr = P / R;  // rank q holds experts [q * epr, (q + 1) * epr)
        if (warp == 0) {
            // receive rows of this block's pairs, in (t, j) order within an
            // expert; each lane sends its pair's row (quantised, or BF16) and
            // scale row to the receive row as soon as it knows it, with TMA
            // bulk stores from shared memory
            const unsigned lt = lanemask_lt();
            const int lo = t0 * k, hi = (t0 + nt) * k;
            const int S = H >> 7;
            for (int c0 = lo; c0 < hi; c0 += 32) {
                const int i = c0 + lane;
                const bool active = i < hi;
                const int p = active ? pp[i] : -2;
                const unsigned peers = __match_any_sync(FULL_MASK, p);
                if (active) {
                    int s = -1;
                    if (p >= 0) {
                        s = run[p] + __popc(peers & lt);
                        a.src[s] = i;
                    }
                    a.slot[i] = s;
                    if (x_ok && (unsigned)s < (unsigned)d.n_rows) {
                        const int tl = (i - lo) / k;
                        if (d.fp8) {
                            bulk_store(d.recv_x + (size_t)s * H, qs + (uint32_t)(tl * H),
                                       (uint32_t)H);
                            if (d.scale_bulk)
                                bulk_store(d.recv_scale + (size_t)s * S,
                                           ss + (uint32_t)(tl * S) * 4u, (uint32_t)S * 4u);
                            else
                                for (int c = 0; c < S; ++c)
                                    d.recv_scale[(size_t)s * S + c] =
                                        reinterpret_cast<const float *>(smem + m.sc_off)[tl * S + c];
                        } else {
                            bulk_store(d.recv_x + (size_t)s * row_bytes,
                                       xs + (uint32_t)tl * row_bytes, row_bytes);
                        }
                    }
                }
                __syncwarp();
                if (active && p >= 0 && (peers & lt) == 0) run[p] += __popc(peers);
                __syncwarp();
            }
            bulk_commit();
            bulk_wait_all();
        } else {
            // meanwhile the other warps write the remaining outputs
            const int w1 = warp - 1, nw = DEC_WARPS - 1;
            // in_rank rows of this block's tokens
            for (int i = tid - 32; i < nt * R; i += DEC_THREADS - 32) {
                const int tl = i / R, q = i - tl * R;
                const int lo = q * epr, hi = lo + epr;
                int hit = 0;
                for (int j = 0; j < k; ++j) {
                    const int p = pp[(t0 + tl) * k + j];
                    hit |= (p >= lo && p < hi);
                }
                a.in_rank[(size_t)(t0 + tl) * R + q] = (uint8_t)hit;
            }
            // the batch-wide arrays, shared out over the blocks: expert p by
            // block p mod NB, rank q by block q mod NB; padding rows of the
            // GEMM layout (src = -1) with their expert
            for (int p = b + NB * (tid - 32); p < P; p += NB * (DEC_THREADS - 32)) {
                a.cnt_expert[p] = hist[p];
                a.expert_off[p] = eoff[p];
            }
            if (b == 0 && tid == 32) {
                a.expert_off[P] = total;
                a.rank_off[R] = total;
            }
            if (A > 1)
                for (int p = b + NB * w1; p < P; p += NB * nw)
                    for (int q = eoff[p] + hist[p] + lane; q < eoff[p + 1]; q += 32) a.src[q] = -1;
            // tokens per rank: a warp per rank, lanes over tokens
            for (int q = b + NB * w1; q < R; q += NB * nw) {
                const int lo = q * epr, hi = lo + epr;
                int cnt = 0;
                for (int tb = 0; tb < T; tb += 32) {  // warp-uniform
                    const int t = tb + lane;
                    int hit = 0;
                    if (t < T)
                        for (int j = 0; j < k; ++j) {
                            const int p = pp[t * k + j];
                            hit |= (p >= lo && p < hi);
                        }
                    cnt += __popc(__ballot_sync(FULL_MASK, hit));
                }
                if (lane == 0) {
                    a.tok_rank[q] = cnt;
                    a.rank_off[q] = eoff[lo];
                    a.rows_rank[q] = eoff[hi] - eoff[lo];
                }
            }
        }
    } else {
        status |= DEV_TIMEOUT_BIT;
    }

    // status bits of all blocks; the last block to leave publishes them
    __syncthreads();
    if (tid == 0) {
        if (status) atomicOr(&d.ctrl[2], status);
        __threadfence();
        if (atomicAdd(&d.ctrl[1], 1) == NB - 1) {
            // every block has left: publish the status and clear the words
            // for the next call (it starts after this grid has finished)
            __threadfence();
            if (a.dev_status != nullptr) *a.dev_status = (int)ld_acquire(&d.ctrl[2]);
            d.ctrl[0] = 0;
            d.ctrl[1] = 0;
            d.ctrl[2] = 0;
        }
    }
}

template <int EPL>
cudaError_t launch_dec(const RouteArgs &r, const LayoutArgs &a, const DecodeArgs &d, int nb,
                       size_t smem, int vec4, cudaStream_t s)
{
    if (smem > 48 * 1024)
        cudaFuncSetAttribute(route_dispatch_small_kernel<EPL>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    return launch_pdl(route_dispatch_small_kernel<EPL>, dim3(nb), dim3(DEC_THREADS), smem, s, r,
                      a, d, vec4);
}

}  // namespace

// tokens per block of the fused kernel for `sms` usable SMs
static int decode_tpb(int T, int sms) { return (T + sms - 1) / sms; }

bool small_route_dispatch_ok(int T, int k, int P, int H, int fp8, int sms)
{
    if (T <= 0 || (long long)T * k > SMALL_MAX_PAIRS || P > SMALL_MAX_PHYS || sms < 1) return false;
    const int tpb = decode_tpb(T, sms);
    // a warp routes one token at a time; up to 8 tokens per block
    if (tpb > DEC_WARPS) return false;
    // the rows of one block are loaded under one mbarrier transaction count
    if ((long long)tpb * 2 * H >= (1 << 20)) return false;
    return decode_smem(tpb, H, fp8, P, T, k).total <= 200 * 1024;
}

cudaError_t launch_route_dispatch_small(const RouteArgs &r, LayoutArgs a, const void *x, int H,
                                        int fp8, int n_rows, void *recv_x, float *recv_scale,
                                        int sms, int *ctrl, uint32_t wait_limit, cudaStream_t s)
{
    const int T = r.T;
    const int tpb = decode_tpb(T, sms);
    const int nb = (T + tpb - 1) / tpb;
    const int S = H / 128;
    DecodeArgs d{static_cast<const uint16_t *>(x), H, fp8, n_rows,
                 static_cast<uint8_t *>(recv_x), recv_scale, tpb,
                 fp8 && (S % 4 == 0) && ((reinterpret_cast<uintptr_t>(recv_scale) & 15) == 0),
                 ctrl, wait_limit};
    const size_t smem = decode_smem(tpb, H, fp8, a.P, T, r.k).total;
    const int vec4 = (r.E % 4 == 0) && ((reinterpret_cast<uintptr_t>(r.logits) & 15) == 0);
    if (r.E <= 32) return launch_dec<1>(r, a, d, nb, smem, vec4, s);
    if (r.E <= 64) return launch_dec<2>(r, a, d, nb, smem, vec4, s);
    if (r.E <= 128) return launch_dec<4>(r, a, d, nb, smem, vec4, s);
    if (r.E <= 256) return launch_dec<8>(r, a, d, nb, smem, vec4, s);
    if (r.E <= 512) return launch_dec<16>(r, a, d, nb, smem, vec4, s);
    return launch_dec<32>(r, a, d, nb, smem, vec4, s);
}

}  // namespace ep
