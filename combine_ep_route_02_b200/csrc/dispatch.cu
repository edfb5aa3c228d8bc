// Dispatch: permute token rows into rank-major, expert-contiguous receive rows,
// optionally quantising each row once to e4m3 with 1x128 block scales before
// writing its k copies.
//
// Per-128-element activation scales computed on the fly from the block's
// maximum absolute value (Perplexity blog, section "Quantization"); FP8
// dispatch with BF16 combine (DeepEP V2 summary, section "Performance").
//
// Mapping: a thread owns a 16-element chunk of a row (32 B of bf16 in, 16 B of
// e4m3 out); the 8 consecutive lanes that own one 128-element block reduce its
// amax with three xor-shuffles.  The row is read once and its quantised bytes
// are stored k times with 16-byte evict-first stores, so the k-fold write
// amplification costs no extra reads or arithmetic.
#include "ep_device.cuh"
#include "ep_internal.h"
#include "quant.cuh"

namespace ep {

namespace {

constexpr int DISPATCH_THREADS = 256;

__global__ void __launch_bounds__(DISPATCH_THREADS)
dispatch_fp8_kernel(const uint16_t *__restrict__ x, int T, int H, int k,
                    const int32_t *__restrict__ slot, uint8_t *__restrict__ recv_x,
                    float *__restrict__ recv_scale, int n_rows)
{
    pdl_launch_dependents();
    pdl_wait();
    const int cpr = H >> 4;  // 16-element chunks per row (a multiple of 8)
    const int S = H >> 7;
    const long long total = (long long)T * cpr;
    const long long stride = (long long)gridDim.x * DISPATCH_THREADS;
    // the loop bound is block-uniform so every lane reaches the shuffles;
    // total is a multiple of 8, so a lane octet is all active or all idle
    const long long g0 = (long long)blockIdx.x * DISPATCH_THREADS + threadIdx.x;
    ChunkWalk it(g0, stride, cpr);
    for (long long base = (long long)blockIdx.x * DISPATCH_THREADS; base < total;
         base += stride, it.next()) {
        const bool active = it.t < T;
        const int t = it.t, c = it.c;
        uint4 lo = make_uint4(0, 0, 0, 0), hi = make_uint4(0, 0, 0, 0);
        if (active) {
            const uint16_t *p = x + (size_t)t * H + (size_t)c * 16;
            lo = ld_stream(p);
            hi = ld_stream(p + 8);
        }
        float scale;
        const uint4 q = quant::quant_chunk(lo, hi, scale);
        if (active) {
            const int32_t *sl = slot + (size_t)t * k;
            for (int j = 0; j < k; ++j) {
                const int s = __ldg(sl + j);
                if ((unsigned)s < (unsigned)n_rows) {
                    st_stream(recv_x + (size_t)s * H + (size_t)c * 16, q);
                    if ((c & 7) == 0) st_stream_f32(recv_scale + (size_t)s * S + (c >> 3), scale);
                }
            }
        }
    }
}

__global__ void __launch_bounds__(DISPATCH_THREADS)
dispatch_bf16_kernel(const uint16_t *__restrict__ x, int T, int H, int k,
                     const int32_t *__restrict__ slot, uint16_t *__restrict__ recv_x, int n_rows)
{
    pdl_launch_dependents();
    pdl_wait();
    const int cpr = H >> 3;  // 8-element (16-byte) chunks per row
    const long long total = (long long)T * cpr;
    const long long g0 = (long long)blockIdx.x * DISPATCH_THREADS + threadIdx.x;
    if (g0 >= total) return;
    ChunkWalk it(g0, (long long)gridDim.x * DISPATCH_THREADS, cpr);
    for (; it.t < T; it.next()) {
        const int t = it.t, c = it.c;
        const uint4 v = ld_stream(x + (size_t)t * H + (size_t)c * 8);
        const int32_t *sl = slot + (size_t)t * k;
        for (int j = 0; j < k; ++j) {
            const int s = __ldg(sl + j);
            if ((unsigned)s < (unsigned)n_rows) st_stream(recv_x + (size_t)s * H + (size_t)c * 8, v);
        }
    }
}

// ---------------------------------------------------------------------------
// FP8 dispatch with TMA bulk copies (rows whose scale row is a whole number of
// 16-byte units, H % 512 == 0).  A persistent CTA walks tokens
// t = blockIdx.x, blockIdx.x + gridDim.x, ...:
//   - thread 0 keeps TMA_IN_STAGES row loads (2H bytes each) in flight into
//     shared memory, each completing on its own mbarrier;
//   - all threads quantise the row from shared memory into an output stage
//     (H code bytes + H/128 fp32 scales);
//   - lanes j < k of warp 0 each send the stage's codes to receive row
//     slot[t, j] with one bulk store and track it in their own bulk group,
//     so an output stage is reused only after its previous stores have read
//     it; meanwhile warps 1.. copy the stage's scale row (H/128 floats) to
//     the k scale rows with ordinary coalesced stores.
// Memory traffic is issued by the TMA engine, so the threads' own loads and
// stores no longer bound the number of bytes in flight.  The engine takes
// its copies one after another at a cost per copy that hardly depends on
// the size, so the small scale rows go by thread stores and each token
// costs k copies, not 2k.
// ---------------------------------------------------------------------------
constexpr int TMA_IN_STAGES = 4;
constexpr int TMA_OUT_STAGES = 4;
constexpr int DEV_TIMEOUT = 4;  // EP_DEV_TIMEOUT

__host__ __device__ inline size_t tma_smem_bytes(int H)
{
    return (size_t)TMA_IN_STAGES * 2 * H + (size_t)TMA_OUT_STAGES * (H + H / 32) +
           TMA_IN_STAGES * sizeof(uint64_t);
}

__global__ void __launch_bounds__(512)
dispatch_fp8_tma_kernel(const uint16_t *__restrict__ x, int T, int H, int k,
                        const int32_t *__restrict__ slot, uint8_t *__restrict__ recv_x,
                        float *__restrict__ recv_scale, int n_rows, int32_t *dev_status,
                        uint32_t wait_limit)
{
    extern __shared__ __align__(128) unsigned char smem[];
    const int S = H >> 7;
    const uint32_t in_bytes = 2u * (uint32_t)H;
    const uint32_t in_base = smem_u32(smem);
    const uint32_t q_base = in_base + TMA_IN_STAGES * in_bytes;
    const uint32_t sc_base = q_base + TMA_OUT_STAGES * (uint32_t)H;
    const uint32_t bar_base = sc_base + TMA_OUT_STAGES * (uint32_t)S * 4u;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int first = blockIdx.x, step = gridDim.x;
    const int n_my = (first < T) ? (T - first + step - 1) / step : 0;
    __shared__ int slot_sh[32];  // this token's k receive rows (k <= 32)

    pdl_launch_dependents();
    if (tid == 0) {
        for (int st = 0; st < TMA_IN_STAGES; ++st) mbar_init(bar_base + 8 * st, 1);
        fence_mbar_init();
    }
    __syncthreads();
    pdl_wait();

    if (tid == 0)
        for (int st = 0; st < TMA_IN_STAGES && st < n_my; ++st) {
            const int t = first + st * step;
            mbar_arrive_expect_tx(bar_base + 8 * st, in_bytes);
            bulk_load(in_base + st * in_bytes, x + (size_t)t * H, in_bytes, bar_base + 8 * st);
        }

    const int cpr = H >> 4;
    int failed_at = -1;
    for (int it = 0; it < n_my; ++it) {
        const int t = first + it * step;
        const int st = it % TMA_IN_STAGES;
        const int o = it % TMA_OUT_STAGES;
        int my_slot = -1;
        if (warp == 0 && lane < k) {
            my_slot = __ldg(slot + (size_t)t * k + lane);
            slot_sh[lane] = my_slot;  // read by the scale-row warps below
        }
        const bool ok = mbar_wait(bar_base + 8 * st, (it / TMA_IN_STAGES) & 1, wait_limit);
        if (!__syncthreads_and(ok)) {
            failed_at = it;
            break;
        }
        const uint32_t in = in_base + st * in_bytes;
        const uint32_t qo = q_base + o * (uint32_t)H;
        const uint32_t so = sc_base + o * (uint32_t)S * 4u;
        // cpr is a multiple of 8 and the bound is block-uniform, so every lane
        // reaches the shuffles and lane octets are all active or all idle
        for (int c0 = 0; c0 < cpr; c0 += blockDim.x) {
            const int c = c0 + tid;
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
        fence_proxy_async_smem();
        __syncthreads();  // the input stage is consumed, the output stage written
        if (warp == 0) {
            if (lane == 0 && it + TMA_IN_STAGES < n_my) {
                const int t2 = first + (it + TMA_IN_STAGES) * step;
                mbar_arrive_expect_tx(bar_base + 8 * st, in_bytes);
                bulk_load(in, x + (size_t)t2 * H, in_bytes, bar_base + 8 * st);
            }
            if (lane < k) {
                if ((unsigned)my_slot < (unsigned)n_rows)
                    bulk_store(recv_x + (size_t)my_slot * H, qo, (uint32_t)H);
                bulk_commit();
                // the stage written next iteration was sent TMA_OUT_STAGES-1
                // groups ago: wait until those stores have read it
                bulk_wait_read<TMA_OUT_STAGES - 1>();
            }
        } else {
            // scale row j by warp 1 + (j mod (warps - 1)), lanes over its
            // H/128 floats
            const int nw = (int)(blockDim.x >> 5) - 1;
            for (int j = warp - 1; j < k; j += nw) {
                const int sj = slot_sh[j];
                if ((unsigned)sj < (unsigned)n_rows)
                    for (int c = lane; c < S; c += 32) {
                        float v;
                        asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(so + 4u * c));
                        st_stream_f32(recv_scale + (size_t)sj * S + c, v);
                    }
            }
        }
        __syncthreads();
    }
    if (warp == 0 && lane < k) bulk_wait_all();
    if (failed_at >= 0 && tid == 0) {
        // let the loads still in flight land before the CTA's shared memory
        // goes away (with the default limit, whatever limit gave up), then
        // report
        for (int it = failed_at; it < n_my && it < failed_at + TMA_IN_STAGES; ++it)
            mbar_wait(bar_base + 8 * (it % TMA_IN_STAGES), (it / TMA_IN_STAGES) & 1,
                      WAIT_LIMIT_DEFAULT);
        if (dev_status != nullptr) atomicOr(dev_status, DEV_TIMEOUT);
    }
}

int tma_threads(int H)
{
    int t = ((H / 16 + 31) / 32) * 32;
    if (t < 64) t = 64;
    if (t > 512) t = 512;
    return t;
}

}  // namespace

bool dispatch_tma_ok(const DispatchArgs &a)
{
    return a.fp8 && a.H % 512 == 0 && tma_smem_bytes(a.H) <= 200 * 1024 &&
           (reinterpret_cast<uintptr_t>(a.recv_scale) & 15) == 0 && a.k <= 32;
}

int dispatch_tma_blocks_per_sm(int H)
{
    const size_t smem = tma_smem_bytes(H);
    cudaFuncSetAttribute(dispatch_fp8_tma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)smem);
    int n = 0;
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, dispatch_fp8_tma_kernel, tma_threads(H), smem);
    return n > 0 ? n : 1;
}

int dispatch_blocks_per_sm(int fp8)
{
    int n = 0;
    if (fp8)
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, dispatch_fp8_kernel, DISPATCH_THREADS, 0);
    else
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, dispatch_bf16_kernel, DISPATCH_THREADS, 0);
    return n > 0 ? n : 1;
}

cudaError_t launch_dispatch(const DispatchArgs &a, cudaStream_t s)
{
    if (a.T == 0) return cudaSuccess;
    if (a.tma_grid > 0) {
        const int blocks = a.T < a.tma_grid ? a.T : a.tma_grid;
        return launch_pdl(dispatch_fp8_tma_kernel, dim3(blocks), dim3(tma_threads(a.H)),
                          tma_smem_bytes(a.H), s, static_cast<const uint16_t *>(a.x), a.T, a.H,
                          a.k, a.slot, static_cast<uint8_t *>(a.recv_x), a.recv_scale,
                          a.n_rows, a.dev_status, a.wait_limit);
    }
    const long long chunks = (long long)a.T * (a.fp8 ? a.H / 16 : a.H / 8);
    long long blocks = (chunks + DISPATCH_THREADS - 1) / DISPATCH_THREADS;
    if (blocks > a.grid) blocks = a.grid;
    const int n_rows = a.n_rows;
    if (a.fp8)
        return launch_pdl(dispatch_fp8_kernel, dim3((int)blocks), dim3(DISPATCH_THREADS), 0, s,
                          static_cast<const uint16_t *>(a.x), a.T, a.H, a.k, a.slot,
                          static_cast<uint8_t *>(a.recv_x), a.recv_scale, n_rows);
    return launch_pdl(dispatch_bf16_kernel, dim3((int)blocks), dim3(DISPATCH_THREADS), 0, s,
                      static_cast<const uint16_t *>(a.x), a.T, a.H, a.k, a.slot,
                      static_cast<uint16_t *>(a.recv_x), n_rows);
}

}  // namespace ep
