// C-ABI entry points of libep_b200: host-side argument checks, launch
// configuration, and the mapping of CUDA errors to ep_status.
#include <atomic>

#include "../../include/ep.h"
#include "../../include/ep_testing.h"
#include "ep_internal.h"

namespace ep {

namespace {
std::atomic<long long> g_wait_limit{-1};  // < 0: the default
}  // namespace

uint32_t wait_limit()
{
    const long long v = g_wait_limit.load(std::memory_order_relaxed);
    return v < 0 ? WAIT_LIMIT_DEFAULT : (uint32_t)v;
}

int device_sm_count()
{
    static volatile int cache[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (dev < 64 && cache[dev] > 0) return cache[dev];
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
        n = 148;
    if (dev < 64) cache[dev] = n;
    return n;
}

namespace {

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

ep_status from_cuda(cudaError_t e) { return e == cudaSuccess ? EP_OK : EP_ERR_CUDA; }

// grid of a streaming kernel: num_sms SMs (0 = all) x resident blocks per SM
int streaming_grid(int num_sms, int blocks_per_sm)
{
    const int sms = device_sm_count();
    const int use = (num_sms <= 0 || num_sms > sms) ? sms : num_sms;
    return use * blocks_per_sm;
}

int cached_blocks_per_sm(int which)
{
    // which: 0 = dispatch bf16, 1 = dispatch fp8, 2 = combine
    static volatile int cache[64][3] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && cache[dev][which] > 0) return cache[dev][which];
    const int n = which == 2 ? combine_blocks_per_sm() : dispatch_blocks_per_sm(which);
    if (dev < 64) cache[dev][which] = n;
    return n;
}

// TMA dispatch CTAs per SM for row length H (depends on shared memory)
int tma_blocks_per_sm(int H)
{
    static volatile int cache_h[64] = {0};
    static volatile int cache_n[64] = {0};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && cache_h[dev] == H && cache_n[dev] > 0) return cache_n[dev];
    const int n = dispatch_tma_blocks_per_sm(H);
    if (dev < 64) {
        cache_n[dev] = n;
        cache_h[dev] = H;
    }
    return n;
}

}  // namespace
}  // namespace ep

using namespace ep;

extern "C" {

const char *ep_status_string(ep_status s)
{
    switch (s) {
    case EP_OK: return "EP_OK";
    case EP_ERR_INVALID: return "EP_ERR_INVALID: invalid argument";
    case EP_ERR_UNSUPPORTED: return "EP_ERR_UNSUPPORTED: size above a library limit";
    case EP_ERR_CUDA: return "EP_ERR_CUDA: CUDA launch or API error";
    case EP_ERR_DEVICE: return "EP_ERR_DEVICE: bad data reported by the device";
    }
    return "unknown ep_status";
}

size_t ep_workspace_size(int T, int k, int P, int R)
{
    if (T < 0 || k < 1 || P < 1 || R < 1) return 0;
    return layout_workspace_bytes(T, k, P, R);
}

}  // extern "C"

namespace ep {
namespace {

ep_status check_route(const float *logits, const float *bias, int T, ep_route_cfg cfg,
                      int32_t *topk_idx, float *topk_w)
{
    const int E = cfg.num_experts, G = cfg.n_group, Kg = cfg.topk_group, k = cfg.topk;
    if (T < 0 || E < 1 || G < 1 || Kg < 1 || k < 1) return EP_ERR_INVALID;
    if (E % G != 0 || Kg > G || (G > 1 && E / G < 2)) return EP_ERR_INVALID;
    if ((long long)k > (long long)(E / G) * Kg) return EP_ERR_INVALID;
    if (E > MAX_EXPERTS || G > MAX_GROUPS || k > MAX_TOPK) return EP_ERR_UNSUPPORTED;
    if ((long long)T * E >= (1LL << 31) || (long long)T * k >= (1LL << 31)) return EP_ERR_UNSUPPORTED;
    if (T > 0 && (!logits || !topk_idx || !topk_w)) return EP_ERR_INVALID;
    if (!aligned(logits, 4) || !aligned(bias, 4) || !aligned(topk_idx, 4) || !aligned(topk_w, 4))
        return EP_ERR_INVALID;
    return EP_OK;
}

ep_status check_layout(const int32_t *topk_idx, int T, int k, int E, int P, int R,
                       const int32_t *phys_of, const int32_t *n_rep, int max_rep, int row_align,
                       int32_t *cnt_expert, int32_t *expert_off, int32_t *rows_rank,
                       int32_t *rank_off, int32_t *tok_rank, uint8_t *in_rank, int32_t *slot,
                       int32_t *src, void *workspace, int32_t *dev_status)
{
    if (T < 0 || k < 1 || E < 1 || P < 1 || R < 1) return EP_ERR_INVALID;
    if (P % R != 0) return EP_ERR_INVALID;
    if ((phys_of == nullptr) != (n_rep == nullptr)) return EP_ERR_INVALID;
    if (phys_of == nullptr && P != E) return EP_ERR_INVALID;
    if (phys_of != nullptr && (P < E || max_rep < 1)) return EP_ERR_INVALID;
    if (k > MAX_TOPK || P > MAX_PHYS) return EP_ERR_UNSUPPORTED;
    if (row_align < 1) return EP_ERR_INVALID;
    if (row_align > MAX_ROW_ALIGN) return EP_ERR_UNSUPPORTED;
    if ((long long)T * k >= (1LL << 31) || (long long)T * R >= (1LL << 31)) return EP_ERR_UNSUPPORTED;
    if ((long long)T * k + (long long)P * (row_align - 1) >= (1LL << 31)) return EP_ERR_UNSUPPORTED;
    if (!cnt_expert || !expert_off || !rows_rank || !rank_off || !tok_rank) return EP_ERR_INVALID;
    if (T > 0 && (!topk_idx || !in_rank || !slot || !src || !workspace)) return EP_ERR_INVALID;
    if (!aligned(workspace, 256) || !aligned(topk_idx, 4) || !aligned(slot, 4) || !aligned(src, 4) ||
        !aligned(dev_status, 4))
        return EP_ERR_INVALID;
    return EP_OK;
}

// receive rows of a copy call: recv_rows, or T * k when recv_rows <= 0
int rows_of(int recv_rows, int T, int k) { return recv_rows > 0 ? recv_rows : T * k; }

LayoutArgs layout_args(const int32_t *topk_idx, int T, int k, int E, int P, int R,
                       const int32_t *phys_of, const int32_t *n_rep, int max_rep, int row_align,
                       int32_t *cnt_expert, int32_t *expert_off, int32_t *rows_rank,
                       int32_t *rank_off, int32_t *tok_rank, uint8_t *in_rank, int32_t *slot,
                       int32_t *src, void *workspace, int32_t *dev_status)
{
    const int NT = layout_tiles(T, k, P);
    char *ws = static_cast<char *>(workspace);
    const size_t o1 = align256((size_t)NT * P * sizeof(int32_t));
    const size_t o2 = o1 + align256((size_t)NT * R * sizeof(int32_t));
    return LayoutArgs{topk_idx, T, k, E, P, R, phys_of, n_rep, max_rep,
                      cnt_expert, expert_off, rows_rank, rank_off, tok_rank, in_rank, slot, src,
                      reinterpret_cast<int32_t *>(ws), reinterpret_cast<int32_t *>(ws + o1),
                      reinterpret_cast<int32_t *>(ws + o2), dev_status,
                      layout_tile_tokens(T, k, P), NT, layout_hist_warps(P), row_align};
}

}  // namespace
}  // namespace ep

extern "C" {

ep_status ep_route(const float *logits, const float *bias, int T, ep_route_cfg cfg,
                   int32_t *topk_idx, float *topk_w, ep_stream_t stream)
{
    EP_TRACE("ep_route");
    const ep_status st = check_route(logits, bias, T, cfg, topk_idx, topk_w);
    if (st != EP_OK) return st;
    RouteArgs a{logits, bias, T, cfg.num_experts, cfg.n_group, cfg.topk_group, cfg.topk,
                cfg.routed_scale, cfg.renorm != 0, topk_idx, topk_w};
    return from_cuda(launch_route(a, reinterpret_cast<cudaStream_t>(stream)));
}

ep_status ep_dispatch_layout(const int32_t *topk_idx, int T, int k, int E, int P, int R,
                             const int32_t *phys_of, const int32_t *n_rep, int max_rep,
                             int row_align, int32_t *cnt_expert, int32_t *expert_off,
                             int32_t *rows_rank, int32_t *rank_off, int32_t *tok_rank,
                             uint8_t *in_rank, int32_t *slot, int32_t *src, void *workspace,
                             int32_t *dev_status, ep_stream_t stream)
{
    EP_TRACE("ep_dispatch_layout");
    const ep_status st = check_layout(topk_idx, T, k, E, P, R, phys_of, n_rep, max_rep, row_align,
                                      cnt_expert, expert_off, rows_rank, rank_off, tok_rank,
                                      in_rank, slot, src, workspace, dev_status);
    if (st != EP_OK) return st;
    const LayoutArgs a = layout_args(topk_idx, T, k, E, P, R, phys_of, n_rep, max_rep, row_align,
                                     cnt_expert, expert_off, rows_rank, rank_off, tok_rank,
                                     in_rank, slot, src, workspace, dev_status);
    return from_cuda(launch_layout(a, reinterpret_cast<cudaStream_t>(stream)));
}

ep_status ep_route_layout(const float *logits, const float *bias, int T, ep_route_cfg cfg,
                          int P, int R, const int32_t *phys_of, const int32_t *n_rep,
                          int max_rep, int row_align, int32_t *topk_idx, float *topk_w,
                          int32_t *cnt_expert, int32_t *expert_off, int32_t *rows_rank,
                          int32_t *rank_off,
                          int32_t *tok_rank, uint8_t *in_rank, int32_t *slot, int32_t *src,
                          void *workspace, int32_t *dev_status, ep_stream_t stream)
{
    EP_TRACE("ep_route_layout");
    ep_status st = check_route(logits, bias, T, cfg, topk_idx, topk_w);
    if (st != EP_OK) return st;
    const int E = cfg.num_experts, k = cfg.topk;
    st = check_layout(topk_idx, T, k, E, P, R, phys_of, n_rep, max_rep, row_align, cnt_expert,
                      expert_off, rows_rank, rank_off, tok_rank, in_rank, slot, src, workspace,
                      dev_status);
    if (st != EP_OK) return st;
    const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const RouteArgs r{logits, bias, T, E, cfg.n_group, cfg.topk_group, k, cfg.routed_scale,
                      cfg.renorm != 0, topk_idx, topk_w};
    const LayoutArgs a = layout_args(topk_idx, T, k, E, P, R, phys_of, n_rep, max_rep, row_align,
                                     cnt_expert, expert_off, rows_rank, rank_off, tok_rank,
                                     in_rank, slot, src, workspace, dev_status);
    if (small_route_layout_ok(T, k, P)) {
        int *done = reinterpret_cast<int *>(static_cast<char *>(workspace) +
                                            layout_workspace_core(T, k, P, R));
        return from_cuda(launch_route_layout_small(r, a, done, s));
    }
    const cudaError_t e = launch_route(r, s);
    if (e != cudaSuccess) return EP_ERR_CUDA;
    return from_cuda(launch_layout(a, s));
}

ep_status ep_dispatch(const void *x_bf16, int T, int H, int k, int recv_rows,
                      const int32_t *slot, int fp8, void *recv_x, float *recv_scale, int num_sms,
                      int32_t *dev_status, ep_stream_t stream)
{
    EP_TRACE("ep_dispatch");
    if (T < 0 || H < 1 || k < 1) return EP_ERR_INVALID;
    if (fp8 ? (H % 128 != 0) : (H % 8 != 0)) return EP_ERR_INVALID;
    if (k > MAX_TOPK) return EP_ERR_UNSUPPORTED;
    if ((long long)T * k >= (1LL << 31) || T > (1 << 30)) return EP_ERR_UNSUPPORTED;
    if (T > 0 && (!x_bf16 || !slot || !recv_x || (fp8 && !recv_scale))) return EP_ERR_INVALID;
    if (!aligned(x_bf16, 16) || !aligned(recv_x, 16) || !aligned(recv_scale, 4) || !aligned(slot, 4) ||
        !aligned(dev_status, 4))
        return EP_ERR_INVALID;
    DispatchArgs a{x_bf16, T, H, k, slot, fp8 != 0, recv_x, recv_scale,
                   streaming_grid(num_sms, cached_blocks_per_sm(fp8 != 0)), 0, dev_status,
                   rows_of(recv_rows, T, k), wait_limit()};
    if (T > 0 && dispatch_tma_ok(a)) a.tma_grid = streaming_grid(num_sms, tma_blocks_per_sm(H));
    return from_cuda(launch_dispatch(a, reinterpret_cast<cudaStream_t>(stream)));
}

ep_status ep_route_dispatch(const float *logits, const float *bias, int T, ep_route_cfg cfg,
                            int P, int R, const int32_t *phys_of, const int32_t *n_rep,
                            int max_rep, int row_align, const void *x_bf16, int H, int fp8,
                            int recv_rows, void *recv_x, float *recv_scale, int32_t *topk_idx,
                            float *topk_w, int32_t *cnt_expert, int32_t *expert_off,
                            int32_t *rows_rank, int32_t *rank_off, int32_t *tok_rank,
                            uint8_t *in_rank, int32_t *slot, int32_t *src, void *workspace,
                            int num_sms, int32_t *dev_status, ep_stream_t stream)
{
    EP_TRACE("ep_route_dispatch");
    ep_status st = check_route(logits, bias, T, cfg, topk_idx, topk_w);
    if (st != EP_OK) return st;
    const int E = cfg.num_experts, k = cfg.topk;
    st = check_layout(topk_idx, T, k, E, P, R, phys_of, n_rep, max_rep, row_align, cnt_expert,
                      expert_off, rows_rank, rank_off, tok_rank, in_rank, slot, src, workspace,
                      dev_status);
    if (st != EP_OK) return st;
    if (H < 1 || (fp8 ? (H % 128 != 0) : (H % 8 != 0))) return EP_ERR_INVALID;
    if (T > (1 << 30)) return EP_ERR_UNSUPPORTED;
    if (T > 0 && (!x_bf16 || !recv_x || (fp8 && !recv_scale))) return EP_ERR_INVALID;
    if (!aligned(x_bf16, 16) || !aligned(recv_x, 16) || !aligned(recv_scale, 4))
        return EP_ERR_INVALID;
    const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const int n_rows = rows_of(recv_rows, T, k);
    const int sms_all = device_sm_count();
    const int sms = (num_sms <= 0 || num_sms > sms_all) ? sms_all : num_sms;
    if (small_route_dispatch_ok(T, k, P, H, fp8 != 0, sms)) {
        const RouteArgs r{logits, bias, T, E, cfg.n_group, cfg.topk_group, k, cfg.routed_scale,
                          cfg.renorm != 0, topk_idx, topk_w};
        const LayoutArgs a = layout_args(topk_idx, T, k, E, P, R, phys_of, n_rep, max_rep,
                                         row_align, cnt_expert, expert_off, rows_rank, rank_off,
                                         tok_rank, in_rank, slot, src, workspace, dev_status);
        // the fused kernel's counters: 64 bytes into the workspace tail (the
        // first bytes of the tail are the small-batch layout's counter)
        int *ctrl = reinterpret_cast<int *>(static_cast<char *>(workspace) +
                                            layout_workspace_core(T, k, P, R) + 64);
        return from_cuda(launch_route_dispatch_small(r, a, x_bf16, H, fp8 != 0, n_rows, recv_x,
                                                     recv_scale, sms, ctrl, wait_limit(), s));
    }
    // larger batches: the two calls' kernels back to back
    st = ep_route_layout(logits, bias, T, cfg, P, R, phys_of, n_rep, max_rep, row_align, topk_idx,
                         topk_w, cnt_expert, expert_off, rows_rank, rank_off, tok_rank, in_rank,
                         slot, src, workspace, dev_status, stream);
    if (st != EP_OK) return st;
    return ep_dispatch(x_bf16, T, H, k, n_rows, slot, fp8, recv_x, recv_scale, num_sms,
                       dev_status, stream);
}

ep_status ep_testing_set_wait_limit(long long polls)
{
    EP_TRACE("ep_testing_set_wait_limit");
    if (polls > 0xffffffffLL) return EP_ERR_INVALID;
    g_wait_limit.store(polls < 0 ? -1 : polls, std::memory_order_relaxed);
    return EP_OK;
}

ep_status ep_combine(const void *y_bf16, const int32_t *slot, const float *topk_w, int T, int H,
                     int k, int recv_rows, void *out_bf16, int num_sms, int32_t *dev_status,
                     ep_stream_t stream)
{
    EP_TRACE("ep_combine");
    if (T < 0 || H < 1 || k < 1 || H % 8 != 0) return EP_ERR_INVALID;
    if (k > MAX_TOPK) return EP_ERR_UNSUPPORTED;
    if ((long long)T * k >= (1LL << 31) || T > (1 << 30)) return EP_ERR_UNSUPPORTED;
    if (T > 0 && (!y_bf16 || !slot || !topk_w || !out_bf16)) return EP_ERR_INVALID;
    if (!aligned(y_bf16, 16) || !aligned(out_bf16, 16) || !aligned(slot, 4) || !aligned(topk_w, 4) ||
        !aligned(dev_status, 4))
        return EP_ERR_INVALID;
    CombineArgs a{y_bf16, slot, topk_w, T, H, k, out_bf16,
                  streaming_grid(num_sms, cached_blocks_per_sm(2)), rows_of(recv_rows, T, k)};
    return from_cuda(launch_combine(a, reinterpret_cast<cudaStream_t>(stream)));
}

ep_status ep_dispatch_backward(const void *grad_recv_bf16, const int32_t *slot, int T, int H,
                               int k, int recv_rows, void *grad_x_bf16, int num_sms,
                               int32_t *dev_status, ep_stream_t stream)
{
    EP_TRACE("ep_dispatch_backward");
    if (T < 0 || H < 1 || k < 1 || H % 8 != 0) return EP_ERR_INVALID;
    if (k > MAX_TOPK) return EP_ERR_UNSUPPORTED;
    if ((long long)T * k >= (1LL << 31) || T > (1 << 30)) return EP_ERR_UNSUPPORTED;
    if (T > 0 && (!grad_recv_bf16 || !slot || !grad_x_bf16)) return EP_ERR_INVALID;
    if (!aligned(grad_recv_bf16, 16) || !aligned(grad_x_bf16, 16) || !aligned(slot, 4) ||
        !aligned(dev_status, 4))
        return EP_ERR_INVALID;
    CombineArgs a{grad_recv_bf16, slot, nullptr, T, H, k, grad_x_bf16,
                  streaming_grid(num_sms, cached_blocks_per_sm(2)), rows_of(recv_rows, T, k)};
    return from_cuda(launch_combine(a, reinterpret_cast<cudaStream_t>(stream)));
}

ep_status ep_combine_backward(const void *grad_out_bf16, const void *y_bf16, const int32_t *slot,
                              const float *topk_w, int T, int H, int k, int recv_rows,
                              void *grad_y_bf16, float *grad_w, int num_sms, int32_t *dev_status,
                              ep_stream_t stream)
{
    EP_TRACE("ep_combine_backward");
    if (T < 0 || H < 1 || k < 1 || H % 8 != 0) return EP_ERR_INVALID;
    if (k > MAX_TOPK) return EP_ERR_UNSUPPORTED;
    if ((long long)T * k >= (1LL << 31) || T > (1 << 30)) return EP_ERR_UNSUPPORTED;
    if (T > 0 && (!grad_out_bf16 || !y_bf16 || !slot || !topk_w || !grad_y_bf16 || !grad_w))
        return EP_ERR_INVALID;
    if (!aligned(grad_out_bf16, 16) || !aligned(y_bf16, 16) || !aligned(grad_y_bf16, 16) ||
        !aligned(slot, 4) || !aligned(topk_w, 4) || !aligned(grad_w, 4) || !aligned(dev_status, 4))
        return EP_ERR_INVALID;
    static volatile int occ[64] = {0};
    int dev = 0;
    cudaGetDevice(&dev);
    int per_sm = dev < 64 ? occ[dev] : 0;
    if (per_sm <= 0) {
        per_sm = combine_backward_blocks_per_sm();
        if (dev < 64) occ[dev] = per_sm;
    }
    CombineBackwardArgs a{grad_out_bf16, y_bf16, slot, topk_w, T, H, k, grad_y_bf16, grad_w,
                          streaming_grid(num_sms, per_sm), rows_of(recv_rows, T, k)};
    return from_cuda(launch_combine_backward(a, reinterpret_cast<cudaStream_t>(stream)));
}

ep_status ep_silu_mul(const void *gate_up_bf16, int n_rows, int I, const int32_t *expert_off,
                      const int32_t *cnt_expert, int P, int fp8, void *act, float *act_scale,
                      int num_sms, ep_stream_t stream)
{
    EP_TRACE("ep_silu_mul");
    if (n_rows < 0 || I < 1 || I % 128 != 0) return EP_ERR_INVALID;
    if ((expert_off == nullptr) != (cnt_expert == nullptr)) return EP_ERR_INVALID;
    if (expert_off != nullptr && P < 1) return EP_ERR_INVALID;
    if (P > MAX_PHYS) return EP_ERR_UNSUPPORTED;
    if ((long long)n_rows * 2 * I >= (1LL << 40)) return EP_ERR_UNSUPPORTED;
    if (n_rows > 0 && (!gate_up_bf16 || !act || (fp8 && !act_scale))) return EP_ERR_INVALID;
    if (!aligned(gate_up_bf16, 16) || !aligned(act, 16) || !aligned(act_scale, 4) ||
        !aligned(expert_off, 4) || !aligned(cnt_expert, 4))
        return EP_ERR_INVALID;
    static volatile int occ[64] = {0};
    int dev = 0;
    cudaGetDevice(&dev);
    int per_sm = dev < 64 ? occ[dev] : 0;
    if (per_sm <= 0) {
        per_sm = activation_blocks_per_sm();
        if (dev < 64) occ[dev] = per_sm;
    }
    ActivationArgs a{gate_up_bf16, n_rows, I, expert_off, cnt_expert, expert_off ? P : 0,
                     fp8 != 0, act, act_scale, streaming_grid(num_sms, per_sm)};
    return from_cuda(launch_activation(a, reinterpret_cast<cudaStream_t>(stream)));
}

}  // extern "C"
