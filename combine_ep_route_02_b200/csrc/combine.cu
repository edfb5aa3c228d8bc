// Combine: top-k weighted gather-reduce of expert output rows back to token
// order, fp32 accumulation, one BF16 rounding at the end.
//
// Expert outputs return to the source token and are summed with the top-k
// weights (Perplexity blog, section "Expert Parallelism"); the combine runs
// in BF16 (DeepEP V2 summary, section "Performance").
//
// Mapping: a thread owns an 8-element (16-byte) chunk of one output row and
// issues all k row loads of that chunk before it accumulates, so k * 16 B per
// thread are in flight; rows are streamed past L1.
#include "ep_device.cuh"
#include "ep_internal.h"

namespace ep {

namespace {

constexpr int COMBINE_THREADS = 256;
constexpr int COMBINE_BATCH = 8;  // row loads issued together

__global__ void __launch_bounds__(COMBINE_THREADS)
combine_kernel(const uint16_t *__restrict__ y, const int32_t *__restrict__ slot,
               const float *__restrict__ w, int T, int H, int k, int n_rows,
               uint16_t *__restrict__ out)
{
    pdl_launch_dependents();
    pdl_wait();
    const int cpr = H >> 3;
    const long long total = (long long)T * cpr;
    const long long g0 = (long long)blockIdx.x * COMBINE_THREADS + threadIdx.x;
    if (g0 >= total) return;
    ChunkWalk it(g0, (long long)gridDim.x * COMBINE_THREADS, cpr);
    for (; it.t < T; it.next()) {
        const int t = it.t, c = it.c;
        float acc[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] = 0.0f;
        for (int j0 = 0; j0 < k; j0 += COMBINE_BATCH) {
            uint4 v[COMBINE_BATCH];
            float wj[COMBINE_BATCH];
            bool ok[COMBINE_BATCH];
#pragma unroll
            for (int u = 0; u < COMBINE_BATCH; ++u) {
                const int j = j0 + u;
                const int s = (j < k) ? __ldg(slot + (size_t)t * k + j) : -1;
                ok[u] = (unsigned)s < (unsigned)n_rows;
                // w == nullptr: unit weights (the dispatch backward); the
                // product by 1 is exact, so the sum is the plain fp32 sum
                wj[u] = ok[u] ? (w != nullptr ? __ldg(w + (size_t)t * k + j) : 1.0f) : 0.0f;
                v[u] = ok[u] ? ld_stream(y + (size_t)s * H + (size_t)c * 8) : make_uint4(0, 0, 0, 0);
            }
            // fp32 accumulation in j order: acc = RN(acc + RN(w * y)); the
            // _rn intrinsics are never fused into an FMA
#pragma unroll
            for (int u = 0; u < COMBINE_BATCH; ++u) {
                if (!ok[u]) continue;
                const uint32_t p[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
                for (int m = 0; m < 4; ++m) {
                    acc[2 * m] = __fadd_rn(acc[2 * m], __fmul_rn(wj[u], bf16_lo(p[m])));
                    acc[2 * m + 1] = __fadd_rn(acc[2 * m + 1], __fmul_rn(wj[u], bf16_hi(p[m])));
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

}  // namespace

int combine_blocks_per_sm()
{
    int n = 0;
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, combine_kernel, COMBINE_THREADS, 0);
    return n > 0 ? n : 1;
}

cudaError_t launch_combine(const CombineArgs &a, cudaStream_t s)
{
    if (a.T == 0) return cudaSuccess;
    const long long chunks = (long long)a.T * (a.H / 8);
    long long blocks = (chunks + COMBINE_THREADS - 1) / COMBINE_THREADS;
    if (blocks > a.grid) blocks = a.grid;
    return launch_pdl(combine_kernel, dim3((int)blocks), dim3(COMBINE_THREADS), 0, s,
                      static_cast<const uint16_t *>(a.y), a.slot, a.w, a.T, a.H, a.k, a.n_rows,
                      static_cast<uint16_t *>(a.out));
}

}  // namespace ep
