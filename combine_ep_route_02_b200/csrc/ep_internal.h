// Internal launch interface between the C-ABI layer (ep_api.cu) and the
// kernel translation units.  Not installed; callers use include/ep.h.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace ep {

// Tokens per tile of the layout kernels.  The workspace size depends on it.
constexpr int LAYOUT_TILE = 64;
constexpr int LAYOUT_THREADS = 256;
constexpr int LAYOUT_WARPS = LAYOUT_THREADS / 32;
constexpr int MAX_EXPERTS = 1024;   // logical experts (routing)
constexpr int MAX_PHYS = 4096;      // physical experts (layout)
constexpr int MAX_TOPK = 32;
constexpr int MAX_GROUPS = 32;

struct RouteArgs {
    const float *logits;
    const float *bias;
    int T, E, G, Kg, k;
    float scale;
    int renorm;
    int32_t *topk_idx;
    float *topk_w;
};

struct LayoutArgs {
    const int32_t *topk_idx;
    int T, k, E, P, R;
    const int32_t *phys_of;
    const int32_t *n_rep;
    int max_rep;
    int32_t *cnt_expert, *expert_off, *rows_rank, *rank_off, *tok_rank;
    uint8_t *in_rank;
    int32_t *slot, *src;
    int32_t *tile_cnt;  // workspace [NT][P]
    int32_t *tile_tok;  // workspace [NT][R]
    int32_t *dev_status;
};

struct DispatchArgs {
    const void *x;
    int T, H, k;
    const int32_t *slot;
    int fp8;
    void *recv_x;
    float *recv_scale;
    int grid;
};

struct CombineArgs {
    const void *y;
    const int32_t *slot;
    const float *w;
    int T, H, k;
    void *out;
    int grid;
};

inline int layout_tiles(int T) { return (T + LAYOUT_TILE - 1) / LAYOUT_TILE; }

cudaError_t launch_route(const RouteArgs &a, cudaStream_t s);
cudaError_t launch_layout(const LayoutArgs &a, cudaStream_t s);
cudaError_t launch_dispatch(const DispatchArgs &a, cudaStream_t s);
cudaError_t launch_combine(const CombineArgs &a, cudaStream_t s);

// resident blocks per SM for each streaming kernel at its block size
int dispatch_blocks_per_sm(int fp8);
int combine_blocks_per_sm();
int device_sm_count();

}  // namespace ep
