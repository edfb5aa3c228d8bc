// Expert activation between the two grouped GEMMs of a gated-SiLU expert:
// h = silu(gate) * up for the rows the routing counts say are filled, then
// 1x128 block quantisation of h to e4m3 for the second GEMM.
//
// The Perplexity blog (section "Quantization") describes this kernel: the
// SiLU has to work under CUDA graphs, with block quantisation and with a
// token count that only the routing knows, so a fixed number of persistent
// blocks read the per-expert counts on the device and share out the filled
// rows among themselves instead of sizing the launch from the buffer.
//
// Arithmetic (exact, so the result does not depend on the schedule):
//   s = bf16(silu(g)), silu(g) = g / (1 + e^-g) correctly rounded
//   h = bf16(fp32(s * u))
//   then the dispatch quantiser on h (quant.cuh).
// The correctly rounded SiLU is a function of the 16-bit gate pattern: a
// table generated at build time (gen_silu_table.c) holds it for all 65,536
// patterns, NaN, infinities and the closed-form ranges included, and each
// block copies it (128 KB) into shared memory, where a lookup indexed by the
// raw gate bits costs one shared load and no range test.  Every entry is
// checked against the oracle on the host, and every gate through the kernel
// on the GPU.
//
// Mapping: one block of 768 threads per SM (the table leaves room for one),
// so 24 warps keep loads in flight.  The filled rows are numbered v = 0 ..
// V-1 in expert order (V = sum of the counts) and each block takes a
// contiguous range of them; a thread
// owns a 16-element chunk of one output row (two 16-byte loads of gate, two
// of up, one 16-byte store of e4m3), and the 8 lanes of a 128-element block
// reduce its amax with shuffles.  Each block keeps the counts' prefix sum in
// shared memory; a thread finds its first chunk's expert by binary search
// and then walks forward.  The next chunk's loads are issued before the
// current chunk is computed.
#include "ep_device.cuh"
#include "ep_internal.h"
#include "quant.cuh"

namespace ep {

namespace {

constexpr int ACT_THREADS = 768;

// silu(g) correctly rounded to bf16 for every bf16 gate pattern g (entry g),
// generated at build time (gen_silu_table.c).
constexpr int TAB_SIZE = 65536;
__device__ const uint16_t kSiluTable[TAB_SIZE] = {
#include "silu_table.inc"
};

// bf16x2 product rounded once to nearest even.  s and u have 8-bit
// significands, so s * u is exact in fp32 wherever bf16 rounding can give a
// nonzero result, and this equals bf16(fp32(s * u)).
EP_DEV uint32_t mul_bf16x2(uint32_t a, uint32_t b)
{
    uint32_t r;
    asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

// h for the 8 elements of one 16-byte gate vector and one 16-byte up vector:
// both halves of each packed gate pair index the table directly.
EP_DEV uint4 silu_mul8(uint4 g, uint4 u, const uint16_t *tab)
{
    const uint32_t gp[4] = {g.x, g.y, g.z, g.w};
    const uint32_t up[4] = {u.x, u.y, u.z, u.w};
    uint32_t h[4];
#pragma unroll
    for (int m = 0; m < 4; ++m) {
        const uint32_t s = __byte_perm((uint32_t)tab[gp[m] & 0xFFFFu], (uint32_t)tab[gp[m] >> 16],
                                       0x5410);
        h[m] = mul_bf16x2(s, up[m]);
    }
    return make_uint4(h[0], h[1], h[2], h[3]);
}

// Filled row number v -> buffer row: expert p is the last one with cum[p] <=
// v (experts with no rows share their cum value with the next one and are
// passed over).  A thread's v only grows, so p is found once by binary search
// and then walked forward.
EP_DEV int first_expert(const int *cum, int P, int v)
{
    int lo = 0, hi = P;  // cum[lo] <= v < cum[hi]
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (cum[mid] <= v) lo = mid;
        else hi = mid;
    }
    return lo;
}

EP_DEV int filled_row(const int *cum, const int *eoff, int &p, int v)
{
    while (cum[p + 1] <= v) ++p;  // cum[P] = V > v ends the walk
    return eoff[p] + (v - cum[p]);
}

// One 16-element chunk in flight: chunk c of buffer row `row`.  A lane whose
// chunk index is past the block's range (or whose row lies outside the
// buffer) is inactive and holds zeros: it still takes part in the shuffles
// but stores nothing (its whole octet is inactive with it).
struct Chunk {
    uint4 g0, g1, u0, u1;
    int row, c;
    bool active;
};

EP_DEV void fetch_chunk(Chunk &ch, const uint16_t *__restrict__ gate_up, int n_rows, int I,
                        const int *cum, const int *eoff, int &p, bool counted, long long base,
                        long long total, const ChunkWalk &it)
{
    ch.g0 = ch.g1 = ch.u0 = ch.u1 = make_uint4(0, 0, 0, 0);
    ch.row = ch.c = 0;
    ch.active = base + threadIdx.x < total;
    if (ch.active) {
        ch.row = counted ? filled_row(cum, eoff, p, it.t) : it.t;
        ch.c = it.c;
        ch.active = (unsigned)ch.row < (unsigned)n_rows;  // offsets beyond the buffer: skipped
    }
    if (ch.active) {
        const uint16_t *gp = gate_up + (size_t)ch.row * 2 * I + (size_t)ch.c * 16;
        ch.g0 = ld_stream(gp);
        ch.g1 = ld_stream(gp + 8);
        ch.u0 = ld_stream(gp + I);
        ch.u1 = ld_stream(gp + I + 8);
    }
}

template <bool FP8>
EP_DEV void process_chunk(const Chunk &ch, const uint16_t *tab, int I, void *act,
                          float *act_scale)
{
    const uint4 h0 = silu_mul8(ch.g0, ch.u0, tab);
    const uint4 h1 = silu_mul8(ch.g1, ch.u1, tab);
    if (FP8) {
        float scale;
        const uint4 q = quant::quant_chunk(h0, h1, scale);
        if (ch.active) {
            st_stream(static_cast<uint8_t *>(act) + (size_t)ch.row * I + (size_t)ch.c * 16, q);
            if ((ch.c & 7) == 0) st_stream_f32(act_scale + (size_t)ch.row * (I >> 7) + (ch.c >> 3), scale);
        }
    } else if (ch.active) {
        uint16_t *o = static_cast<uint16_t *>(act) + (size_t)ch.row * I + (size_t)ch.c * 16;
        st_stream(o, h0);
        st_stream(o + 8, h1);
    }
}

template <bool FP8>
__global__ void __launch_bounds__(ACT_THREADS)
silu_mul_kernel(const uint16_t *__restrict__ gate_up, int n_rows, int I,
                const int32_t *__restrict__ expert_off, const int32_t *__restrict__ cnt_expert,
                int P, void *__restrict__ act, float *__restrict__ act_scale)
{
    extern __shared__ __align__(16) int sm[];
    uint16_t *tab = reinterpret_cast<uint16_t *>(sm);  // [TAB_SIZE] the SiLU table
    int *cum = sm + TAB_SIZE / 2;  // [P + 1]  prefix sum of the counts
    int *eoff = cum + P + 1;       // [P]      first buffer row of each expert
    __shared__ int warp_tot[ACT_THREADS / 32 + 1];
    pdl_launch_dependents();
    // the table is no input of this call: copy it while the previous kernel
    // finishes
    for (int i = threadIdx.x; i < TAB_SIZE / 8; i += blockDim.x)
        reinterpret_cast<uint4 *>(tab)[i] = reinterpret_cast<const uint4 *>(kSiluTable)[i];
    pdl_wait();

    int V = n_rows;
    const bool counted = expert_off != nullptr;
    if (counted) {
        const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
        // block-wide exclusive scan of the counts, ACT_THREADS at a time
        int carry = 0;
        for (int base = 0; base < P; base += ACT_THREADS) {
            const int p = base + threadIdx.x;
            const int c = p < P ? cnt_expert[p] : 0;
            if (p < P) eoff[p] = expert_off[p];
            const int incl = warp_inclusive_scan(c);
            if (lane == 31) warp_tot[warp] = incl;
            __syncthreads();
            if (warp == 0) {
                const int wt = lane < ACT_THREADS / 32 ? warp_tot[lane] : 0;
                const int wi = warp_inclusive_scan(wt);
                if (lane < ACT_THREADS / 32) warp_tot[lane] = wi - wt;
                if (lane == ACT_THREADS / 32 - 1) warp_tot[ACT_THREADS / 32] = wi;
            }
            __syncthreads();
            if (p < P) cum[p] = carry + warp_tot[warp] + incl - c;
            carry += warp_tot[ACT_THREADS / 32];
            __syncthreads();
        }
        if (threadIdx.x == 0) cum[P] = carry;
        V = min(carry, n_rows);
    }
    __syncthreads();  // table and prefix sums complete

    const int cpr = I >> 4;        // 16-element chunks per output row (multiple of 8)
    // each block takes a contiguous range of filled rows, so a thread's
    // expert index moves forward by at most one expert per row it crosses
    const long long rows_per_block = ((long long)V + gridDim.x - 1) / gridDim.x;
    const long long v0 = min((long long)V, (long long)blockIdx.x * rows_per_block);
    const long long v1 = min((long long)V, v0 + rows_per_block);
    const long long total = v1 * cpr;
    const long long stride = ACT_THREADS;
    // block-uniform loop bound so every lane reaches the shuffles; the range
    // starts and ends on row boundaries (cpr is a multiple of 8), so a lane
    // octet is all active or all idle
    long long base = v0 * cpr;
    ChunkWalk it(base + threadIdx.x, stride, cpr);
    int p = (counted && base + threadIdx.x < total) ? first_expert(cum, P, it.t) : 0;
    Chunk cur;
    fetch_chunk(cur, gate_up, n_rows, I, cum, eoff, p, counted, base, total, it);
    while (base < total) {
        // issue the next chunk's loads before computing this one
        ChunkWalk nit = it;
        nit.next();
        Chunk nxt;
        fetch_chunk(nxt, gate_up, n_rows, I, cum, eoff, p, counted, base + stride, total, nit);
        process_chunk<FP8>(cur, tab, I, act, act_scale);
        cur = nxt;
        it = nit;
        base += stride;
    }
}

size_t act_smem_bytes(int P)
{
    return sizeof(uint16_t) * TAB_SIZE + sizeof(int) * (size_t)(2 * P + 1);
}

}  // namespace

// Called once per device before the first launch there: opts both instances
// in to the shared memory of the largest expert count (128 KB of table plus
// 32 KB of prefix sums at MAX_PHYS experts).
int activation_blocks_per_sm()
{
    const int most = (int)act_smem_bytes(MAX_PHYS);
    cudaFuncSetAttribute(silu_mul_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, most);
    cudaFuncSetAttribute(silu_mul_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, most);
    int n = 0;
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, silu_mul_kernel<true>, ACT_THREADS,
                                                  act_smem_bytes(256));
    return n > 0 ? n : 1;
}

cudaError_t launch_activation(const ActivationArgs &a, cudaStream_t s)
{
    if (a.n_rows == 0) return cudaSuccess;
    const int P = a.expert_off != nullptr ? a.P : 0;
    const size_t smem = act_smem_bytes(P);
    // without counts the work is known on the host: no more blocks than chunks
    long long blocks = a.grid;
    if (a.expert_off == nullptr) {
        const long long chunks = (long long)a.n_rows * (a.I / 16);
        const long long need = (chunks + ACT_THREADS - 1) / ACT_THREADS;
        if (need < blocks) blocks = need;
    }
    if (a.fp8)
        return launch_pdl(silu_mul_kernel<true>, dim3((int)blocks), dim3(ACT_THREADS), smem, s,
                          static_cast<const uint16_t *>(a.gate_up), a.n_rows, a.I, a.expert_off,
                          a.cnt_expert, P, a.act, a.act_scale);
    return launch_pdl(silu_mul_kernel<false>, dim3((int)blocks), dim3(ACT_THREADS), smem, s,
                      static_cast<const uint16_t *>(a.gate_up), a.n_rows, a.I, a.expert_off,
                      a.cnt_expert, P, a.act, a.act_scale);
}

}  // namespace ep
