// Allocation-free dispatch layout.
//
// ep_dispatch_layout needs a small device scratch buffer (per-tile expert
// histograms and per-tile rank counts).  Some callers cannot hand one over:
// code that runs inside another runtime's enqueue hook (an inference-engine
// plugin, a framework operator with no access to its caching allocator) may
// not allocate device memory at that point, and cudaMalloc can synchronise
// the whole device, which a latency-bound decode step cannot afford.  For
// them this file keeps the scratch in a fixed-size __device__ array that
// lives as long as the library is loaded, and forwards to the ordinary entry
// point with that array as the workspace.
#include <mutex>

#include "../../include/ep.h"
#include "ep_internal.h"

namespace {

// Fixed scratch, one copy per GPU that loads the library, held until exit.
__device__ __align__(256) unsigned char g_layout_scratch[EP_NOALLOC_SCRATCH_BYTES];

std::mutex g_scratch_mu;
void *g_scratch_addr[64] = {};  // device address of g_layout_scratch, per device

// Host code cannot use &g_layout_scratch (that is a host-side shadow, not a
// device address); the runtime gives the real address once per device.
cudaError_t scratch_address(void **out)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (g_scratch_addr[dev] == nullptr) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_layout_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return cudaSuccess;
}

}  // namespace

extern "C" ep_status ep_dispatch_layout_noalloc(
    const int32_t *topk_idx, int T, int k, int E, int P, int R, const int32_t *phys_of,
    const int32_t *n_rep, int max_rep, int32_t *cnt_expert, int32_t *expert_off,
    int32_t *rows_rank, int32_t *rank_off, int32_t *tok_rank, uint8_t *in_rank, int32_t *slot,
    int32_t *src, int32_t *dev_status, ep_stream_t stream)
{
    EP_TRACE("ep_dispatch_layout_noalloc");
    const size_t need = ep_workspace_size(T, k, P, R);
    if (need == 0) return EP_ERR_INVALID;
    if (need > EP_NOALLOC_SCRATCH_BYTES) return EP_ERR_UNSUPPORTED;
    void *scratch = nullptr;
    if (scratch_address(&scratch) != cudaSuccess) return EP_ERR_CUDA;
    // the layout kernels overwrite every scratch word they read, so the
    // previous call's contents need no clearing
    return ep_dispatch_layout(topk_idx, T, k, E, P, R, phys_of, n_rep, max_rep, 1, cnt_expert,
                              expert_off, rows_rank, rank_off, tok_rank, in_rank, slot, src,
                              scratch, dev_status, stream);
}
