// Internal launch interface between the C-ABI layer (ep_api.cu) and the
// kernel translation units.  Not installed; callers use include/ep.h.
#pragma once

#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>
#include <stdint.h>

namespace ep {

// A named NVTX range around each entry point (shows up in Nsight Systems
// timelines; without an attached tool the calls return at once).
struct NvtxRange {
    explicit NvtxRange(const char *name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
    NvtxRange(const NvtxRange &) = delete;
    NvtxRange &operator=(const NvtxRange &) = delete;
};
#define EP_TRACE(name) ::ep::NvtxRange ep_nvtx_range_(name)

// Layout tiling.  A tile of tokens is one block of the count and slot
// kernels.  Up to LAYOUT_FUSED_MAX_TILES tiles, the slot kernel sums the tile
// histograms of its expert columns itself; above that a column-scan kernel
// runs in between.  The workspace size depends on this tiling.
constexpr int LAYOUT_MIN_TILE = 64;
constexpr int LAYOUT_MAX_TILE = 512;
constexpr int LAYOUT_FUSED_MAX_TILES = 64;
constexpr int LAYOUT_THREADS = 1024;
constexpr int LAYOUT_WARPS = LAYOUT_THREADS / 32;
constexpr int MAX_EXPERTS = 1024;   // logical experts (routing)
constexpr int MAX_PHYS = 4096;      // physical experts (layout)
constexpr int MAX_TOPK = 32;
constexpr int MAX_GROUPS = 32;
constexpr int MAX_ROW_ALIGN = 1024;  // GEMM row tile of the padded layout

// Polls a bounded device-side wait makes before it gives up and reports
// EP_DEV_TIMEOUT (a wait for a TMA copy, or for the other blocks of a grid).
// wait_limit() is this default unless a failure-detection test changed it
// (ep_testing_set_wait_limit); waits that drain copies still in flight after
// a give-up always use the default.
constexpr uint32_t WAIT_LIMIT_DEFAULT = 1u << 22;
uint32_t wait_limit();

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
    int32_t *tile_bad;  // workspace [NT]: status bits found by each count block
    int32_t *dev_status;
    int tile_tokens;    // TT
    int n_tiles;        // NT
    int hist_warps;     // slot-kernel warps that order pairs
    int row_align;      // each expert's first receive row is a multiple of this
};

struct DispatchArgs {
    const void *x;
    int T, H, k;
    const int32_t *slot;
    int fp8;
    void *recv_x;
    float *recv_scale;
    int grid;          // register-path grid
    int tma_grid;      // > 0: use the TMA pipeline with this many CTAs
    int32_t *dev_status;
    int n_rows;        // receive rows; slots outside [0, n_rows) are skipped
    uint32_t wait_limit;  // polls of each bounded TMA wait
};

struct CombineArgs {
    const void *y;
    const int32_t *slot;
    const float *w;
    int T, H, k;
    void *out;
    int grid;
    int n_rows;        // rows of y; slots outside [0, n_rows) are skipped
};

// Warps of the slot kernel that each order one contiguous share of a tile's
// pairs (each keeps a P-entry table in shared memory): 32, or fewer for
// large P so that the tables stay within 128 KB.
inline int layout_hist_warps(int P)
{
    int w = LAYOUT_WARPS;
    while (w > 1 && (size_t)w * P > 32768) w >>= 1;
    return w;
}

// Tokens per tile: enough for at most LAYOUT_FUSED_MAX_TILES tiles, within
// [LAYOUT_MIN_TILE, LAYOUT_MAX_TILE], and small enough that the slot kernel's
// shared memory ((2 P + 1) + hist_warps * P ints of tables + tile_tokens * k
// ints of pair ids) stays under 200 KB.
inline int layout_tile_tokens(int T, int k, int P)
{
    int tt = (T + LAYOUT_FUSED_MAX_TILES - 1) / LAYOUT_FUSED_MAX_TILES;
    if (tt < LAYOUT_MIN_TILE) tt = LAYOUT_MIN_TILE;
    if (tt > LAYOUT_MAX_TILE) tt = LAYOUT_MAX_TILE;
    int cap = (51200 - (2 * P + 1) - layout_hist_warps(P) * P) / (k > 0 ? k : 1);
    cap = (cap / 32) * 32;
    if (cap < 32) cap = 32;
    return tt < cap ? tt : cap;
}
inline int layout_tiles(int T, int k, int P)
{
    const int tt = layout_tile_tokens(T, k, P);
    return (T + tt - 1) / tt;
}
struct CombineBackwardArgs {
    const void *g;     // grad_out bf16 [T, H]
    const void *y;     // expert rows bf16 [T*k, H]
    const int32_t *slot;
    const float *w;
    int T, H, k;
    void *grad_y;      // bf16 [n_rows, H]
    float *grad_w;     // [T, k]
    int grid;
    int n_rows;        // rows of y and grad_y
};

// Expert activation: h = silu(gate) * up over the rows the per-expert counts
// select, quantised to e4m3 with 1x128 scales (or stored as bf16).
struct ActivationArgs {
    const void *gate_up;       // bf16 [n_rows, 2I]
    int n_rows, I;
    const int32_t *expert_off; // [P+1] or null (every row)
    const int32_t *cnt_expert; // [P]
    int P;
    int fp8;
    void *act;                 // e4m3 [n_rows, I] or bf16 [n_rows, I]
    float *act_scale;          // [n_rows, I/128] when fp8
    int grid;
};

inline size_t align256(size_t n) { return (n + 255) & ~size_t(255); }
// workspace bytes: tile_cnt, tile_tok, tile_bad, each 256-byte aligned, then
// 256 bytes: the small-batch layout kernel's completion counter at +0 and the
// route + dispatch kernel's counters at +64
inline size_t layout_workspace_core(int T, int k, int P, int R)
{
    const size_t NT = (size_t)layout_tiles(T > 0 ? T : 1, k, P);
    return align256(NT * P * sizeof(int32_t)) + align256(NT * R * sizeof(int32_t)) +
           align256(NT * sizeof(int32_t));
}
inline size_t layout_workspace_bytes(int T, int k, int P, int R)
{
    return layout_workspace_core(T, k, P, R) + 256;
}

// Fused routing + layout for small batches (one kernel; see fused.cu).
constexpr int SMALL_MAX_PAIRS = 4096;
constexpr int SMALL_MAX_PHYS = 1024;

// Programmatic dependent launch: every kernel of the path is launched with
// programmatic stream serialisation, calls pdl_launch_dependents() so the
// next kernel's launch can begin, and pdl_wait() before it touches global
// memory, which returns once the previous kernel in the stream has finished
// and its writes are visible.  Without the launch attribute both are no-ops.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t s, Args... args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

cudaError_t launch_route(const RouteArgs &a, cudaStream_t s);
bool small_route_layout_ok(int T, int k, int P);
cudaError_t launch_route_layout_small(const RouteArgs &r, LayoutArgs a, int *done,
                                      cudaStream_t s);
// Fused routing + layout + dispatch for small batches (one kernel; see
// decode.cu).  ctrl: 4 ints of workspace, zero before the first launch and
// left zero by every launch.
bool small_route_dispatch_ok(int T, int k, int P, int H, int fp8, int sms);
cudaError_t launch_route_dispatch_small(const RouteArgs &r, LayoutArgs a, const void *x, int H,
                                        int fp8, int n_rows, void *recv_x, float *recv_scale,
                                        int sms, int *ctrl, uint32_t wait_limit, cudaStream_t s);
cudaError_t launch_layout(const LayoutArgs &a, cudaStream_t s);
cudaError_t launch_dispatch(const DispatchArgs &a, cudaStream_t s);
cudaError_t launch_combine(const CombineArgs &a, cudaStream_t s);
cudaError_t launch_combine_backward(const CombineBackwardArgs &a, cudaStream_t s);
int combine_backward_blocks_per_sm();
cudaError_t launch_activation(const ActivationArgs &a, cudaStream_t s);
int activation_blocks_per_sm();

// resident blocks per SM for each streaming kernel at its block size
int dispatch_blocks_per_sm(int fp8);
bool dispatch_tma_ok(const DispatchArgs &a);
int dispatch_tma_blocks_per_sm(int H);
int combine_blocks_per_sm();
int device_sm_count();

}  // namespace ep
