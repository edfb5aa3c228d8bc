// Device helpers shared by the sm_100a kernels of libep_b200.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#define EP_DEV __device__ __forceinline__

namespace ep {

constexpr unsigned FULL_MASK = 0xffffffffu;

// 16-byte streaming load of read-only data: not kept in L1 (every byte is
// read once), L2 prefetch of the surrounding 256 B (rows are contiguous).
EP_DEV uint4 ld_stream(const void *p)
{
    uint4 v;
    asm("ld.global.nc.L1::no_allocate.L2::256B.v4.u32 {%0,%1,%2,%3}, [%4];"
        : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
        : "l"(p));
    return v;
}

// 16-byte store with the evict-first (streaming) policy.
EP_DEV void st_stream(void *p, uint4 v)
{
    asm volatile("st.global.cs.v4.u32 [%0], {%1,%2,%3,%4};" ::"l"(p), "r"(v.x), "r"(v.y),
                 "r"(v.z), "r"(v.w)
                 : "memory");
}

EP_DEV void st_stream_f32(float *p, float v)
{
    asm volatile("st.global.cs.f32 [%0], %1;" ::"l"(p), "f"(v) : "memory");
}

// bf16 pair (low half = lower address) -> two fp32, exact.
EP_DEV float bf16_lo(uint32_t u) { return __uint_as_float(u << 16); }
EP_DEV float bf16_hi(uint32_t u) { return __uint_as_float(u & 0xffff0000u); }

// two fp32 -> packed bf16x2, round to nearest even (lo in the low half).
EP_DEV uint32_t pack_bf16x2(float lo, float hi)
{
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// two fp32 -> packed e4m3x2, round to nearest even, saturating to +-448
// (lo in the low byte).
EP_DEV uint32_t pack_e4m3x2(float lo, float hi)
{
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

// Walks a flat chunk index g = t * cpr + c forward by a fixed stride without
// dividing in the loop: one division when the walk starts.
struct ChunkWalk {
    int t, c, st, sc, cpr;
    EP_DEV ChunkWalk(long long g0, long long stride, int cpr_)
        : t((int)(g0 / cpr_)), c((int)(g0 % cpr_)), st((int)(stride / cpr_)),
          sc((int)(stride % cpr_)), cpr(cpr_) {}
    EP_DEV void next()
    {
        c += sc;
        t += st;
        if (c >= cpr) {
            c -= cpr;
            ++t;
        }
    }
};

// (value desc, index asc) total order used by every selection.
EP_DEV bool beats(float va, int ia, float vb, int ib)
{
    return va > vb || (va == vb && ia < ib);
}

// Butterfly arg-max over the warp; every lane ends with the winner.
EP_DEV void warp_argmax(float &v, int &i)
{
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        float ov = __shfl_xor_sync(FULL_MASK, v, off);
        int oi = __shfl_xor_sync(FULL_MASK, i, off);
        if (beats(ov, oi, v, i)) {
            v = ov;
            i = oi;
        }
    }
}

EP_DEV int warp_inclusive_scan(int v)
{
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        int o = __shfl_up_sync(FULL_MASK, v, off);
        if (lane >= off) v += o;
    }
    return v;
}

EP_DEV unsigned lanemask_lt()
{
    unsigned m;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

}  // namespace ep
