// Backward of combine (training).  The DeepEP V2 summary (section "Usage for
// training, prefill and decoding") states that combine's backward is a
// dispatch: every receive row gets its token's output gradient scaled by the
// routing weight, and the routing weights get the dot products of the output
// gradient with the expert rows.
//
//   grad_y[slot[t,j]] = bf16( fp32(w[t,j] * g[t]) )
//   grad_w[t,j]       = sum_h g[t,h] * y[slot[t,j],h]       (fp32)
//
// A block owns one token at a time (persistent over tokens): it reads the
// gradient row once, streams the k expert rows, writes the k scaled rows and
// reduces the k dot products across its warps.  The block has as many
// threads (a multiple of 32, at most 256) as give every thread the same
// number of 8-element chunks of a row (224 for H = 7168), and the kernel is
// compiled for k <= 8 separately so that its partial sums stay in few
// registers (three blocks per SM).
#include "ep_device.cuh"
#include "ep_internal.h"

namespace ep {

namespace {

constexpr int BWD_THREADS = 256;
constexpr int BWD_WARPS = BWD_THREADS / 32;

template <int KMAX>
__global__ void __launch_bounds__(BWD_THREADS, KMAX <= 8 ? 3 : 2)
combine_backward_kernel(const uint16_t *__restrict__ g, const uint16_t *__restrict__ y,
                        const int32_t *__restrict__ slot, const float *__restrict__ w, int T,
                        int H, int k, int n_rows, uint16_t *__restrict__ grad_y,
                        float *__restrict__ grad_w)
{
    __shared__ int s_slot[MAX_TOPK];
    __shared__ float s_w[MAX_TOPK];
    __shared__ float s_part[BWD_WARPS][MAX_TOPK];
    pdl_launch_dependents();
    pdl_wait();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int nthreads = blockDim.x, nwarps = nthreads >> 5;
    const int cpr = H >> 3;
    for (int t = blockIdx.x; t < T; t += gridDim.x) {
        if (threadIdx.x < k) {
            const int sl = __ldg(slot + (size_t)t * k + threadIdx.x);
            s_slot[threadIdx.x] = ((unsigned)sl < (unsigned)n_rows) ? sl : -1;
            s_w[threadIdx.x] = __ldg(w + (size_t)t * k + threadIdx.x);
        }
        __syncthreads();
        float part[KMAX];
#pragma unroll
        for (int j = 0; j < KMAX; ++j) part[j] = 0.0f;
        for (int c = threadIdx.x; c < cpr; c += nthreads) {
            const uint4 gv = ld_stream(g + (size_t)t * H + (size_t)c * 8);
            const uint32_t gp[4] = {gv.x, gv.y, gv.z, gv.w};
            float gf[8];
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                gf[2 * m] = bf16_lo(gp[m]);
                gf[2 * m + 1] = bf16_hi(gp[m]);
            }
            // eight expert rows at a time: all loads issued before the
            // first store (the stores are compiler barriers)
#pragma unroll
            for (int j0 = 0; j0 < KMAX; j0 += 8) {
                if (j0 >= k) break;
                uint4 yv[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const int sl = (j0 + u < k) ? s_slot[j0 + u] : -1;
                    yv[u] = sl >= 0 ? ld_stream(y + (size_t)sl * H + (size_t)c * 8)
                                    : make_uint4(0, 0, 0, 0);
                }
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const int j = j0 + u;
                    if (j >= k) break;
                    const int sl = s_slot[j];
                    if (sl < 0) continue;
                    const uint32_t yp[4] = {yv[u].x, yv[u].y, yv[u].z, yv[u].w};
                    const float wj = s_w[j];
                    uint4 o;
                    uint32_t *op = reinterpret_cast<uint32_t *>(&o);
                    float acc = part[j];
#pragma unroll
                    for (int m = 0; m < 4; ++m) {
                        acc = fmaf(gf[2 * m], bf16_lo(yp[m]), acc);
                        acc = fmaf(gf[2 * m + 1], bf16_hi(yp[m]), acc);
                        op[m] = pack_bf16x2(__fmul_rn(wj, gf[2 * m]), __fmul_rn(wj, gf[2 * m + 1]));
                    }
                    part[j] = acc;
                    st_stream(grad_y + (size_t)sl * H + (size_t)c * 8, o);
                }
            }
        }
        // reduce each dot product over the block
#pragma unroll
        for (int j = 0; j < KMAX; ++j) {
            if (j >= k) break;
            float v = part[j];
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(FULL_MASK, v, off);
            if (lane == 0) s_part[warp][j] = v;
        }
        __syncthreads();
        if (threadIdx.x < k) {
            float v = 0.0f;
#pragma unroll
            for (int q = 0; q < nwarps; ++q) v += s_part[q][threadIdx.x];
            grad_w[(size_t)t * k + threadIdx.x] = (s_slot[threadIdx.x] >= 0) ? v : 0.0f;
        }
        __syncthreads();  // s_slot / s_w / s_part are rewritten for the next token
    }
}

}  // namespace

cudaError_t launch_combine_backward(const CombineBackwardArgs &a, cudaStream_t s)
{
    if (a.T == 0) return cudaSuccess;
    const int blocks = a.T < a.grid ? a.T : a.grid;
    // threads per block: the fewest multiples of 32 (up to BWD_THREADS) that
    // give every thread the same number of 8-element chunks of a row
    const int cpr = a.H / 8;
    const int per = (cpr + BWD_THREADS - 1) / BWD_THREADS;
    int nt = ((cpr + per - 1) / per + 31) / 32 * 32;
    if (nt > BWD_THREADS) nt = BWD_THREADS;
    if (a.k <= 8)
        return launch_pdl(combine_backward_kernel<8>, dim3(blocks), dim3(nt), 0, s,
                          static_cast<const uint16_t *>(a.g), static_cast<const uint16_t *>(a.y),
                          a.slot, a.w, a.T, a.H, a.k, a.n_rows, static_cast<uint16_t *>(a.grad_y),
                          a.grad_w);
    return launch_pdl(combine_backward_kernel<MAX_TOPK>, dim3(blocks), dim3(nt), 0, s,
                      static_cast<const uint16_t *>(a.g), static_cast<const uint16_t *>(a.y),
                      a.slot, a.w, a.T, a.H, a.k, a.n_rows, static_cast<uint16_t *>(a.grad_y),
                      a.grad_w);
}

int combine_backward_blocks_per_sm()
{
    int n = 0;
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, combine_backward_kernel<8>, BWD_THREADS, 0);
    return n > 0 ? n : 1;
}

}  // namespace ep
