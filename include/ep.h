/*
 * ep.h -- C ABI of the B200 (sm_100a) MoE expert-parallel routing, dispatch
 * layout, FP8 dispatch and combine library (libep_b200.so).
 *
 * The operations are the four steps around the experts of a MoE layer:
 *
 *   ep_route            gate logits -> top-k expert ids and weights
 *   ep_dispatch_layout  top-k ids   -> per-expert / per-rank counts, prefix
 *                                      sums, receive-row slots
 *   ep_dispatch         tokens      -> rank-major, expert-contiguous receive
 *                                      rows (BF16 copies, or e4m3 + 1x128
 *                                      scales)
 *   ep_combine          expert rows -> top-k weighted sum per token (BF16)
 *   ep_silu_mul         expert intermediate rows -> silu(gate) * up, e4m3 +
 *                                      1x128 scales for the second expert GEMM
 *
 * Sources (page title, then section):
 *  - Perplexity, "Lower latency and higher throughput with multi-node
 *    DeepSeek deployment": section "Expert Parallelism" (256 routed experts,
 *    8 per token, weighted sum; dispatch and combine are the two all-to-alls
 *    around the experts), section "Quantization" (1x128 activation scales,
 *    M x ceil_div(K,128) of them, amax over 128-element sub-blocks), section
 *    "MoE Router" (Mixtral top-k is DeepSeek group routing with one group;
 *    dense dispatch/combine plans need per-expert aggregates), section
 *    "CUDA Graph" (kernels read the routing counts instead of sizing work from
 *    buffer capacities, so they can be captured).
 *  - DeepEP V2 summary (news.hada.io, "DeepSeek merilis library open source
 *    DeepEP"), section on the ElasticBuffer interface (buffer size hint,
 *    num_sms override) and section "Usage for training, prefill and
 *    decoding" (the dispatch handle carries num_recv_tokens_per_expert_list
 *    for the GEMM; combine reduces expert outputs back to the source; a
 *    cached handle skips the layout in decoding).
 *  - DeepSeek Open Infra day-4 summary, EPLB section (group-limited routing;
 *    redundant experts replicated and placed across GPUs).
 *
 * On one GPU the expert-parallel ranks are logical: rank r owns physical
 * experts [r*P/R, (r+1)*P/R) and its receive rows are the contiguous range
 * [rank_off[r], rank_off[r+1]) of one buffer.
 *
 * Conventions for every entry point
 *  - Memory: every array pointer is DEVICE memory allocated and freed by the
 *    caller.  The library allocates nothing, frees nothing, keeps no state
 *    between calls and never synchronises the host.  All work is enqueued on
 *    `stream` (NULL = the legacy default stream).
 *  - Layout: row-major, densely packed.  Index arrays are int32.
 *  - Errors: argument checks happen on the host before anything is enqueued
 *    and return EP_ERR_INVALID (bad shape / value / alignment) or
 *    EP_ERR_UNSUPPORTED (valid but beyond the library's limits).  A launch
 *    failure returns EP_ERR_CUDA.  Bad data found on the device (an expert id
 *    outside [0,E), an invalid replica map entry) never traps: it sets bits
 *    in the caller's *dev_status and the offending pair gets slot -1.
 *  - Empty input (T == 0) is valid and produces empty / zero outputs.
 */
#ifndef EP_B200_H
#define EP_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    EP_OK = 0,
    EP_ERR_INVALID = 1,     /* bad argument: shape, value, alignment, NULL */
    EP_ERR_UNSUPPORTED = 2, /* valid but above a limit of this library */
    EP_ERR_CUDA = 3,        /* a CUDA launch or API call (or a NCCL call) failed */
    EP_ERR_DEVICE = 4       /* reserved for callers mapping *dev_status */
} ep_status;

/* Bits reported through a caller's *dev_status word. */
#define EP_DEV_BAD_EXPERT 1  /* layout: a topk_idx entry outside [0, E) */
#define EP_DEV_BAD_REPLICA 2 /* layout: n_rep[e] outside [1, max_rep] or phys id outside [0, P) */
#define EP_DEV_TIMEOUT 4     /* dispatch / route_dispatch / peer calls: a bounded wait (for
                                an asynchronous copy, for the other blocks of the grid, or
                                for another rank) gave up; that call's output is incomplete */
#define EP_DEV_OVERFLOW 8    /* peer dispatch: a destination row beyond the receive
                                buffers' capacity (the pair was skipped) */

/* Same object as cudaStream_t; no CUDA header is needed to use this API. */
typedef struct CUstream_st *ep_stream_t;

/* Routing configuration.
 *   num_experts   E, 1..1024
 *   n_group       G: experts form G runs of E/G consecutive ids; 1..32,
 *                 E % G == 0, and E/G >= 2 when G > 1
 *   topk_group    groups kept per token, 1..G
 *   topk          k experts per token, 1..32, k <= (E/G) * topk_group
 *   routed_scale  multiplies every weight (2.5 for DeepSeek-V3)
 *   renorm        nonzero: weights are divided by their sum before scaling */
typedef struct {
    int num_experts;
    int n_group;
    int topk_group;
    int topk;
    float routed_scale;
    int renorm;
} ep_route_cfg;

/*
 * Bytes of device scratch that ep_dispatch_layout needs for T tokens, top-k,
 * P physical experts and R logical ranks (the counterpart of DeepEP's buffer
 * size hint).  Returns 0 for invalid sizes.  The scratch need not be zeroed
 * for the layout calls; ep_route_dispatch wants it zeroed once (see there).
 */
size_t ep_workspace_size(int T, int k, int P, int R);

/*
 * Sigmoid-gated, group-limited top-k routing (DeepSeek-V3 style; EPLB
 * section of the DeepSeek Open Infra summary, MoE Router section of the
 * Perplexity blog).
 *
 *   logits    fp32 [T, E]
 *   bias      fp32 [E] selection bias, or NULL for none
 *   topk_idx  int32 [T, k] (out)  chosen expert ids in selection order
 *   topk_w    fp32  [T, k] (out)  weights
 *
 * Per token: s_e = fp32(1/(1+exp(-x_e))) evaluated in fp64; key_e = s_e + b_e
 * (fp32).  With G > 1 a group scores the fp32 sum of its two largest keys and
 * only the topk_group best groups stay eligible.  The k largest keys among the
 * eligible experts are chosen, ties to the lower index (groups: ties to the
 * lower group id).  w_j = s_{e_j}; with renorm, w_j /= sum_j w_j (fp32, in j
 * order; skipped when the sum is 0); then w_j *= routed_scale.  Every fp32
 * operation rounds once to nearest even.
 */
ep_status ep_route(const float *logits, const float *bias, int T, ep_route_cfg cfg,
                   int32_t *topk_idx, float *topk_w, ep_stream_t stream);

/*
 * Dispatch layout: counts, prefix sums and deterministic slots (the
 * "handle" of DeepEP V2; num_recv_tokens_per_expert_list = cnt_expert).
 *
 *   topk_idx   int32 [T, k] logical expert ids in [0, E)
 *   E, P, R    logical experts, physical experts, logical ranks; P % R == 0;
 *              P == E unless a replica map is given (then P >= E)
 *   phys_of    int32 [E, max_rep] or NULL: physical ids of each expert's
 *              replicas; token t uses replica phys_of[e][t % n_rep[e]]
 *   n_rep      int32 [E] or NULL (together with phys_of)
 *   row_align  A, 1..1024: the GEMM layout of the DeepEP V2 summary (its
 *              feature list names a new GEMM layout).  Each expert's first
 *              receive row is a multiple of A (the row tile of a grouped GEMM
 *              reading the receive buffer); A = 1 packs the rows.
 *   outputs    cnt_expert [P]     rows per physical expert (pairs, unpadded)
 *              expert_off [P+1]   first row of each expert:
 *                                 expert_off[p+1] = expert_off[p] +
 *                                 round_up(cnt_expert[p], A)
 *              rows_rank  [R]     rows per rank (its experts' padded rows)
 *              rank_off   [R+1]   exclusive prefix sum of rows_rank
 *              tok_rank   [R]     tokens with at least one expert on the rank
 *              in_rank    uint8 [T, R]  1 if token t sends to rank r
 *              slot       [T, k]  receive row of pair (t, j); -1 if invalid
 *              src        [T*k + P*(A-1)] for rows [0, expert_off[P]):
 *                                 src[slot[t,j]] = t*k + j, and -1 for the
 *                                 padding rows that follow each expert's pairs
 *   workspace  ep_workspace_size(T, k, P, R) bytes, 256-byte aligned
 *   dev_status int32 [1] or NULL; zeroed by this call, then EP_DEV_* bits
 *
 * Receive rows are ordered by physical expert, and within an expert by
 * (t, j).  Expert p's pairs fill rows [expert_off[p], expert_off[p] +
 * cnt_expert[p]); with A = 1 there is no padding and valid pairs fill rows
 * [0, expert_off[P]).  A receive buffer of T*k + P*(A-1) rows holds any
 * routing.  Rank r's rows are [rank_off[r], rank_off[r+1]).  The result
 * does not depend on scheduling (no global atomics decide an order).
 * T*k + P*(A-1) >= 2^31 returns EP_ERR_UNSUPPORTED.
 */
ep_status ep_dispatch_layout(const int32_t *topk_idx, int T, int k, int E, int P, int R,
                             const int32_t *phys_of, const int32_t *n_rep, int max_rep,
                             int row_align, int32_t *cnt_expert, int32_t *expert_off,
                             int32_t *rows_rank, int32_t *rank_off, int32_t *tok_rank,
                             uint8_t *in_rank, int32_t *slot, int32_t *src, void *workspace,
                             int32_t *dev_status, ep_stream_t stream);

/*
 * Routing followed by the dispatch layout, in one call (the cached-handle /
 * low-latency decode use of the DeepEP V2 summary, section "Usage for
 * training, prefill and decoding").  Arguments are those of ep_route and
 * ep_dispatch_layout (E = cfg.num_experts, k = cfg.topk); the results are
 * identical to calling the two in sequence.  For small batches
 * (T * k <= 4096 and P <= 1024) a single kernel does both: its routing blocks
 * count themselves done on a counter in the workspace, and the last one lays
 * out the whole batch, so no block waits for another.  Larger batches run the
 * two calls' kernels back to back.  workspace: ep_workspace_size(T, k, P, R)
 * bytes, 256-byte aligned.
 */
ep_status ep_route_layout(const float *logits, const float *bias, int T, ep_route_cfg cfg,
                          int P, int R, const int32_t *phys_of, const int32_t *n_rep,
                          int max_rep, int row_align, int32_t *topk_idx, float *topk_w, int32_t *cnt_expert,
                          int32_t *expert_off, int32_t *rows_rank, int32_t *rank_off,
                          int32_t *tok_rank, uint8_t *in_rank, int32_t *slot, int32_t *src,
                          void *workspace, int32_t *dev_status, ep_stream_t stream);

/*
 * Dispatch (permute, optionally with fused 1x128 FP8 quantisation).
 *
 *   x_bf16      bf16 [T, H], 16-byte aligned; H % 8 == 0 (H % 128 == 0 for fp8)
 *   recv_rows   N, rows of the receive buffer; N <= 0 means T*k (the packed
 *               layout); a padded layout needs up to T*k + P*(row_align-1)
 *   slot        int32 [T, k] from ep_dispatch_layout (or a cached copy)
 *   fp8 == 0:   recv_x is bf16 [N, H]; row slot[t,j] = x[t] bit for bit
 *   fp8 != 0:   recv_x is e4m3fn [N, H] and recv_scale fp32 [N, H/128];
 *               per 128-element block b of x[t]: amax = max|x|, scale =
 *               fp32(amax / 448), q = e4m3_rn_satfinite(fp32(x / scale));
 *               a block with amax == 0 gets scale 0 and zero bytes
 *   num_sms     SMs to spread the work over (0 = all), like DeepEP's num_sms
 *   dev_status  int32 [1] or NULL: EP_DEV_TIMEOUT is ORed in if a bounded
 *               wait on a TMA copy gives up (the word is not cleared here)
 *
 * Slots outside [0, N) are skipped, and rows no slot names (padding) are
 * left as they were.  recv_x must be 16-byte aligned, recv_scale 4-byte aligned.  With
 * fp8, H % 512 == 0 and a 16-byte aligned recv_scale, rows move through
 * shared memory by TMA bulk copies; otherwise by 16-byte thread stores.
 */
ep_status ep_dispatch(const void *x_bf16, int T, int H, int k, int recv_rows,
                      const int32_t *slot, int fp8, void *recv_x, float *recv_scale, int num_sms,
                      int32_t *dev_status, ep_stream_t stream);

/*
 * Routing, dispatch layout and dispatch in one call: the low-latency decode
 * path of the DeepEP V2 summary (section "Usage for training, prefill and
 * decoding"), whose small batches are bound by launches and dependency
 * latency rather than bytes.  Arguments are those of ep_route_layout
 * followed by those of ep_dispatch (x_bf16, H, fp8, recv_rows, recv_x,
 * recv_scale), with E = cfg.num_experts and k = cfg.topk; every output is
 * identical to calling ep_route_layout and then ep_dispatch.  The layout
 * outputs can be reused by later ep_dispatch / ep_combine calls (the cached
 * handle of the same section).
 *
 * For small batches (T * k <= 4096, P <= 1024, at most 8 tokens per SM and
 * the rows of a block within 200 KB of shared memory) one kernel does all
 * three steps with at most one block per SM: each block loads its tokens'
 * rows with TMA, routes them, quantises them while the other blocks route,
 * waits at a grid-wide counter in the workspace (a bounded wait), lays out
 * the whole batch from the T*k ids in L2 and sends its rows to their
 * receive rows.  Larger batches run ep_route_layout's and ep_dispatch's
 * kernels back to back.
 *
 *   num_sms     SMs to use (0 = all): caps the fused kernel's blocks and the
 *               dispatch grid
 *   workspace   ep_workspace_size(T, k, P, R) bytes, 256-byte aligned.
 *               Zero it once before its first use by this call: the fused
 *               kernel counts on 16 bytes of it, and leaves them zero again
 *               when it finishes (after a timeout too), so later calls need
 *               no clearing; the other calls do not touch those bytes.
 *   dev_status  int32 [1] or NULL: zeroed by this call, then the layout's
 *               EP_DEV_BAD_* bits and EP_DEV_TIMEOUT if a bounded wait (for a
 *               TMA copy or for the other blocks) gave up, in which case the
 *               outputs are incomplete
 * Checks and limits are those of ep_route_layout and ep_dispatch.
 */
ep_status ep_route_dispatch(const float *logits, const float *bias, int T, ep_route_cfg cfg,
                            int P, int R, const int32_t *phys_of, const int32_t *n_rep,
                            int max_rep, int row_align, const void *x_bf16, int H, int fp8,
                            int recv_rows, void *recv_x, float *recv_scale, int32_t *topk_idx,
                            float *topk_w, int32_t *cnt_expert, int32_t *expert_off,
                            int32_t *rows_rank, int32_t *rank_off, int32_t *tok_rank,
                            uint8_t *in_rank, int32_t *slot, int32_t *src, void *workspace,
                            int num_sms, int32_t *dev_status, ep_stream_t stream);

/*
 * Combine: weighted gather-reduce back to token order.
 *
 *   y_bf16    bf16 [N, H] expert outputs in receive-row order
 *   slot      int32 [T, k], topk_w fp32 [T, k]
 *   recv_rows N, rows of y (N <= 0 means T*k), as for ep_dispatch
 *   out_bf16  bf16 [T, H] (out)
 *
 * out[t] = bf16_rne( acc ), acc = fp32 sum over j = 0..k-1 in order of
 * fp32(w[t,j] * y[slot[t,j]]), each step rounded to nearest even.  Slots
 * outside [0, N) contribute nothing; padding rows are never read.  y and out 16-byte aligned, H % 8 == 0.
 * dev_status as for ep_dispatch (NULL allowed).
 */
ep_status ep_combine(const void *y_bf16, const int32_t *slot, const float *topk_w, int T,
                     int H, int k, int recv_rows, void *out_bf16, int num_sms,
                     int32_t *dev_status, ep_stream_t stream);

/*
 * Allocation-free variant of ep_dispatch_layout.  It has no counterpart in
 * the pages; it exists for callers that cannot allocate device memory where
 * they call the layout: code running inside another runtime's enqueue hook
 * (an inference-engine plugin, a framework operator without access to its
 * caching allocator), or a latency-bound decode step that cannot afford the
 * device-wide synchronisation cudaMalloc may cause.
 *
 * Arguments and results are those of ep_dispatch_layout with row_align = 1
 * and without `workspace`: the scratch lives in a fixed __device__ array of
 * EP_NOALLOC_SCRATCH_BYTES inside the library, which every GPU that loads
 * the library keeps until the process exits.  Sizes whose
 * ep_workspace_size(T, k, P, R) exceeds that limit return
 * EP_ERR_UNSUPPORTED (with k = 8, P = 256 and R = 8 that is about 2M tokens).
 * The first call on each device looks up the array's device address (host
 * code cannot use the array's name as a device pointer) and keeps it for the
 * life of the process; make that first call before any stream capture.  The
 * kept address does not survive cudaDeviceReset: after a reset of a device,
 * do not call this entry point on it again in the same process.  The call allocates and frees nothing.
 * All calls on a device share the one array and it keeps the last call's
 * contents (the kernels need none of them cleared): calls whose work can
 * overlap on the GPU (different streams, or several host threads) race on
 * it and must be serialised by the caller.
 */
#define EP_NOALLOC_SCRATCH_BYTES (4u << 20)
ep_status ep_dispatch_layout_noalloc(const int32_t *topk_idx, int T, int k, int E, int P, int R,
                                     const int32_t *phys_of, const int32_t *n_rep, int max_rep,
                                     int32_t *cnt_expert, int32_t *expert_off,
                                     int32_t *rows_rank, int32_t *rank_off, int32_t *tok_rank,
                                     uint8_t *in_rank, int32_t *slot, int32_t *src,
                                     int32_t *dev_status, ep_stream_t stream);

/*
 * Backward of dispatch (training): the DeepEP V2 summary (section "Usage for
 * training, prefill and decoding") notes that dispatch's backward is a
 * combine.  grad_x[t] = bf16( sum_j grad_recv[slot[t,j]] ), fp32 in j order:
 * ep_combine with unit weights.  With an FP8 forward dispatch the
 * quantisation is treated as the identity; gradients travel in BF16.
 *   grad_recv_bf16  bf16 [N, H] gradients of the receive rows
 *   recv_rows       N (N <= 0 means T*k), as for ep_combine
 *   grad_x_bf16     bf16 [T, H] (out)
 * Alignment, slot handling and dev_status as for ep_combine.
 */
ep_status ep_dispatch_backward(const void *grad_recv_bf16, const int32_t *slot, int T, int H,
                               int k, int recv_rows, void *grad_x_bf16, int num_sms,
                               int32_t *dev_status, ep_stream_t stream);

/*
 * Backward of combine (training): combine's backward is a dispatch (same
 * section).  For out[t] = sum_j w[t,j] y[slot[t,j]]:
 *   grad_y[slot[t,j]] = bf16( fp32(w[t,j] * grad_out[t]) )   bf16 [N, H]
 *   grad_w[t,j]       = sum_h grad_out[t,h] * y[slot[t,j],h]  fp32 [T, k]
 * with y bf16 [N, H] and N = recv_rows (N <= 0 means T*k).
 * The dot products are accumulated in fp32 in an unspecified order (within
 * about 1e-5 of the sum of |terms| of the exact value).  Rows of invalid
 * slots are not written and their grad_w is 0.  16-byte alignment for the
 * bf16 arrays; dev_status as for ep_combine.
 */
ep_status ep_combine_backward(const void *grad_out_bf16, const void *y_bf16, const int32_t *slot,
                              const float *topk_w, int T, int H, int k, int recv_rows,
                              void *grad_y_bf16, float *grad_w, int num_sms, int32_t *dev_status,
                              ep_stream_t stream);

/*
 * Expert activation between the two grouped GEMMs of a gated-SiLU expert,
 * with the 1x128 FP8 quantisation the second GEMM reads (Perplexity blog,
 * section "Quantization": the SiLU kernel works under CUDA graphs, with
 * block quantisation and a routed token count known only on the device, so
 * a fixed set of persistent blocks reads the per-expert counts and shares
 * out the filled rows).
 *
 *   gate_up_bf16  bf16 [n_rows, 2I]: row r = [gate (I) | up (I)], the first
 *                 GEMM's output in receive-row order; 16-byte aligned
 *   I             intermediate width, I % 128 == 0
 *   expert_off    int32 [P+1] and cnt_expert int32 [P] from
 *                 ep_dispatch_layout (device memory, read by the kernel):
 *                 rows [expert_off[p], expert_off[p] + cnt_expert[p]) are
 *                 processed, padding and unused rows are not touched.  Both
 *                 NULL: every one of the n_rows rows is processed.
 *   fp8 != 0:     act is e4m3fn [n_rows, I] and act_scale fp32 [n_rows, I/128]
 *   fp8 == 0:     act is bf16 [n_rows, I] holding h itself (act_scale unused)
 *
 * Per element: s = bf16(silu(g)) with silu(g) = g / (1 + e^-g) correctly
 * rounded (silu(-inf) = -0); h = bf16(fp32(s * u)), each rounding to nearest
 * even.  Per 128-element block of h: amax = max |h| (NaN ignored), scale =
 * fp32(amax / 448), q = e4m3_rn_satfinite(fp32(h / scale)); amax == 0 gives
 * scale 0 and zero bytes.  Rows from offsets outside [0, n_rows) are skipped.
 * The launch size depends on num_sms only, never on the counts, so the call
 * can be captured in a CUDA graph with the counts changing between replays.
 */
ep_status ep_silu_mul(const void *gate_up_bf16, int n_rows, int I, const int32_t *expert_off,
                      const int32_t *cnt_expert, int P, int fp8, void *act, float *act_scale,
                      int num_sms, ep_stream_t stream);

/*
 * Expert parallelism across processes (one GPU each) over NCCL: the dispatch
 * and combine all-to-alls of the Perplexity blog (section "Expert
 * Parallelism") as grouped NCCL sends and receives of whole rows.  Process
 * rank q of the communicator is expert-parallel rank q: it owns physical
 * experts [q*P/W, (q+1)*P/W), so the layout of every rank is computed with
 * R = W, and rows [rank_off[q], rank_off[q+1]) of its receive buffer are the
 * ones rank q needs.
 *
 * The communicator is the caller's (NCCL's ncclComm_t, for example the one
 * behind a torch.distributed NCCL process group); the work is enqueued on
 * `stream`, and the calls must be made in the same order on every rank.  The
 * library loads NCCL at run time: the NCCL already loaded in the process is
 * used, and EP_ERR_UNSUPPORTED is returned when none can be loaded.  A NCCL
 * call that fails returns EP_ERR_CUDA.  Nothing is allocated.
 *
 * The row counts of the data exchanges are host integers (NCCL takes its
 * sizes on the host), so one layout costs one device-to-host read: after
 * ep_exchange_counts the caller copies recv_counts (and its own rows_rank)
 * to the host and synchronises the stream, then both directions of the
 * exchange reuse those counts.
 */
typedef struct ncclComm *ep_nccl_comm; /* the same object as NCCL's ncclComm_t */

/*
 * Counts of one layout's exchange.  Rank q is sent [rows_rank[q],
 * cnt_expert[q*epr], ..., cnt_expert[q*epr + epr-1]] (epr = P/W), and every
 * rank's message arrives in recv_counts:
 *   rows_rank     int32 [W] this rank's receive rows per destination rank
 *   cnt_expert    int32 [P] this rank's pairs per physical expert
 *   send_scratch  int32 [W, 1 + P/W] device scratch (the packed messages)
 *   recv_counts   int32 [W, 1 + P/W] (out): row s = [rows rank s sends
 *                 here, pairs from s for each of this rank's experts]
 * P must be a multiple of the communicator's size W.
 */
ep_status ep_exchange_counts(ep_nccl_comm comm, const int32_t *rows_rank,
                             const int32_t *cnt_expert, int P, int32_t *send_scratch,
                             int32_t *recv_counts, ep_stream_t stream);

/*
 * Dispatch exchange: rows [sum_{q'<q} send_rows[q'], ... + send_rows[q]) of
 * `rows` go to rank q, and the recv_rows[s] rows from rank s land in `recv`
 * starting at row sum_{s'<s} recv_rows[s'] (in the order the source's
 * layout gave them: by expert, then token).  Rows are row_bytes bytes each,
 * so the e4m3 codes, their fp32 scale rows and BF16 rows all use this call.
 *   send_rows  host int32 [W]: this rank's rows_rank
 *   recv_rows  host int32 [W]: column 0 of recv_counts
 * The rank's own share is copied on the device; send_rows[me] must equal
 * recv_rows[me].
 */
ep_status ep_dispatch_exchange(ep_nccl_comm comm, const void *rows, const int32_t *send_rows,
                               const int32_t *recv_rows, size_t row_bytes, void *recv,
                               ep_stream_t stream);

/*
 * Combine exchange, the reverse of ep_dispatch_exchange: the expert outputs
 * of the rows that came from rank s (rows [sum_{s'<s} recv_rows[s'], ... +
 * recv_rows[s]) of expert_rows) go back to rank s, and the rows returning
 * from rank q land in `back` at the rows this rank sent it, [sum_{q'<q}
 * send_rows[q'], ... + send_rows[q]), ready for ep_combine.  Arguments as
 * for ep_dispatch_exchange.
 */
ep_status ep_combine_exchange(ep_nccl_comm comm, const void *expert_rows,
                              const int32_t *recv_rows, const int32_t *send_rows,
                              size_t row_bytes, void *back, ep_stream_t stream);

/*
 * Expert parallelism over peer memory (NVLink / NVSwitch): the dispatch and
 * combine all-to-alls of the Perplexity blog (section "Expert Parallelism")
 * as direct stores into, and loads from, the other ranks' buffers, with no
 * collective library: the FP8 dispatch quantises each token once and stores
 * its k rows straight into the receive buffers of the ranks that own the
 * experts, and the combine gathers the expert outputs straight from them.
 *
 * W ranks; rank q owns physical experts [q*P/W, (q+1)*P/W).  A process
 * serves ranks rank0 .. rank0 + n_local - 1 on its GPU: one rank per GPU
 * across processes, or several ranks in one process (then the calls below
 * cover all of them in one launch, and n_local must not exceed the SM count,
 * since those blocks wait for one another).  Each rank's tokens are laid
 * out first with ep_dispatch_layout (or ep_route_layout) with R = W and
 * row_align 1; the peer calls read cnt_expert, expert_off, slot and topk_w.
 *
 * Rank q receives, for each of its experts e in order, the rows of source
 * rank 0, then source 1, ..., each source's rows in its own (t, j) order;
 * every expert's rows start on a multiple of row_align (the GEMM layout).
 *
 * Step protocol (every rank makes the same calls in the same order):
 *   ep_peer_counts        all-gather of the per-expert counts through the
 *                         boards; each rank computes where its rows go
 *   ep_peer_dispatch      quantise + store rows to their owners, then tell
 *                         every rank this source is complete
 *   ep_peer_wait_dispatch a rank waits for all sources (before its experts)
 *   (the rank's experts turn recv_x into y)
 *   ep_peer_experts_ready a rank publishes that its y is complete
 *   ep_peer_combine       weighted sum of each token's k rows read from the
 *                         ranks that hold them (waits for their publication)
 * Every wait is bounded: a wait that gives up ORs EP_DEV_TIMEOUT into the
 * rank's dev_status and leaves that step's output incomplete.
 *
 * Buffers (all allocated by the caller).  Rank-indexed tables are DEVICE
 * arrays of W device pointers, entry q being rank q's buffer as this process
 * addresses it (its own allocation for a local rank; on one node, a CUDA IPC
 * mapping of a peer's allocation).  Rank q's buffers: recv_x e4m3 [cap, H],
 * recv_scale fp32 [cap, H/128], y bf16 [cap, H], board int32 [W, P], flags
 * int32 [8] (zeroed once when allocated, then left to the library: they
 * count the steps).  cap must hold every row rank q can receive: the sum of
 * all sources' T*k plus (P/W)*(row_align-1); rows beyond cap are skipped and
 * reported as EP_DEV_OVERFLOW.  No TMA and no multicast is used.
 */
typedef struct {
    int world;                /* W */
    int rank0;                /* first rank served by this process */
    int n_local;              /* ranks served by this process */
    int P;                    /* physical experts, a multiple of W */
    int row_align;            /* expert row tile at the destinations (1..1024) */
    int cap;                  /* rows of every rank's receive buffers */
    void *const *recv_x;      /* [W] -> e4m3 [cap, H] */
    float *const *recv_scale; /* [W] -> fp32 [cap, H/128] */
    const void *const *y;     /* [W] -> bf16 [cap, H], expert outputs in receive order */
    int32_t *const *board;    /* [W] -> int32 [W, P] */
    int32_t *const *flags;    /* [W] -> int32 [8] */
} ep_peer_group;

/* One local rank's own arrays (a device array of n_local of these, in rank
 * order, is passed to the calls). */
typedef struct {
    const void *x;              /* bf16 [T, H] tokens */
    const int32_t *cnt_expert;  /* [P]   from its layout (R = W) */
    const int32_t *expert_off;  /* [P+1] */
    const int32_t *slot;        /* [T, k] */
    const float *topk_w;        /* [T, k] */
    void *out;                  /* bf16 [T, H] (out): combine */
    int32_t *dest_off;          /* [P] (out): first row, at expert p's rank, of this
                                   rank's rows for expert p (-1 after a timeout) */
    int32_t *recv_cnt;          /* [P/W, W] (out): pairs from each source for each of
                                   this rank's experts (for its grouped GEMM) */
    int32_t *recv_rows;         /* [1] (out): rows this rank receives, padding included */
    int32_t *pair_dest;         /* [T, k, 2] (out): (rank, row) holding pair (t, j)'s
                                   row, rank -1 if none; 8-byte aligned */
    int32_t *dev_status;        /* [1] or NULL: EP_DEV_* bits are ORed in */
    int T;                      /* tokens of this rank */
    int reserved;
} ep_peer_rank;

/* k: experts per token (the layouts' top-k); max_T: the largest T of the
 * local ranks.  Also writes every local pair's (rank, row) in pair_dest. */
ep_status ep_peer_counts(ep_peer_group g, const ep_peer_rank *ranks, int k, int max_T,
                         ep_stream_t stream);
/* H % 128 == 0; k <= 32; max_T: the largest T of the local ranks (sizes the grid). */
ep_status ep_peer_dispatch(ep_peer_group g, const ep_peer_rank *ranks, int H, int k,
                           int max_T, ep_stream_t stream);
ep_status ep_peer_wait_dispatch(ep_peer_group g, const ep_peer_rank *ranks, ep_stream_t stream);
ep_status ep_peer_experts_ready(ep_peer_group g, ep_stream_t stream);
/* out[t] = bf16(sum_j fp32(w[t,j] * y_q[row])) in j order, as ep_combine; H % 8 == 0. */
ep_status ep_peer_combine(ep_peer_group g, const ep_peer_rank *ranks, int H, int k, int max_T,
                          ep_stream_t stream);

/* Human-readable name of a status code (static string). */
const char *ep_status_string(ep_status status);

#ifdef __cplusplus
}
#endif

#endif /* EP_B200_H */
