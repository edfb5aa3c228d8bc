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

// ---- TMA bulk copies and mbarriers (sm_90+ PTX, CTA-local, no multicast) ----

EP_DEV uint32_t smem_u32(const void *p) { return (uint32_t)__cvta_generic_to_shared(p); }

EP_DEV void mbar_init(uint32_t bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

// make mbarrier initialisation visible to the async (TMA) proxy
EP_DEV void fence_mbar_init() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }

EP_DEV void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}

// plain arrive (count 1) on a CTA-local mbarrier
EP_DEV void mbar_arrive(uint32_t bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

// Polls the barrier phase at most `limit` times; false if it never completed.
EP_DEV bool mbar_wait(uint32_t bar, uint32_t phase, uint32_t limit)
{
    for (uint32_t i = 0; i < limit; ++i) {
        uint32_t done;
        asm volatile(
            "{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2; "
            "selp.u32 %0, 1, 0, p; }"
            : "=r"(done)
            : "r"(bar), "r"(phase)
            : "memory");
        if (done) return true;
    }
    return false;
}

// global -> this CTA's shared memory, completion counted on `bar` (bytes)
EP_DEV void bulk_load(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar)
{
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
        "l"(src), "r"(bytes), "r"(bar)
        : "memory");
}

// this CTA's shared memory -> global, tracked in the issuing thread's bulk groups
EP_DEV void bulk_store(void *dst, uint32_t src, uint32_t bytes)
{
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst), "r"(src),
                 "r"(bytes)
                 : "memory");
}

EP_DEV void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }

// wait until at most N of this thread's bulk groups still read shared memory
template <int N>
EP_DEV void bulk_wait_read()
{
    asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}

// wait until all of this thread's bulk groups have completed their writes
EP_DEV void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// order this thread's generic-proxy shared-memory writes before later
// async-proxy (TMA) reads of them
EP_DEV void fence_proxy_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

EP_DEV uint4 lds128(uint32_t addr)
{
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(addr));
    return v;
}

EP_DEV void sts128(uint32_t addr, uint4 v)
{
    asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z),
                 "r"(v.w)
                 : "memory");
}

// see launch_pdl in ep_internal.h
EP_DEV void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
EP_DEV void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

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
