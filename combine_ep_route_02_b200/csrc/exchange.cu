// Cross-process expert parallelism: the exchange of whole receive rows
// between ranks (one process and one GPU each) over NCCL.
//
// Dispatch and combine are the two all-to-alls around the experts
// (Perplexity blog, section "Expert Parallelism").  The dispatch layout
// already writes the rows bound for rank q as the contiguous range
// [rank_off[q], rank_off[q+1]) of the receive buffer, so each direction is
// one grouped NCCL send/receive per peer of whole rows, on the caller's
// communicator and stream.  The split sizes are needed on the host, which is
// why the per-destination counts travel first (ep_exchange_counts) and the
// caller reads them back once per layout.
//
// NCCL is loaded at run time (the process that owns the communicator has
// loaded it already), so the library has no link-time dependency on it.
#include <dlfcn.h>
#include <nccl.h>

#include <mutex>

#include "../../include/ep.h"
#include "ep_internal.h"

namespace ep {

namespace {

struct NcclApi {
    ncclResult_t (*group_start)();
    ncclResult_t (*group_end)();
    ncclResult_t (*send)(const void *, size_t, ncclDataType_t, int, ncclComm_t, cudaStream_t);
    ncclResult_t (*recv)(void *, size_t, ncclDataType_t, int, ncclComm_t, cudaStream_t);
    ncclResult_t (*count)(const ncclComm_t, int *);
    ncclResult_t (*user_rank)(const ncclComm_t, int *);
    bool ok;
};

std::once_flag g_nccl_once;
NcclApi g_nccl = {};

// The NCCL the process already has (the one that made the communicator),
// else the one the loader finds.
void load_nccl()
{
    void *h = dlopen("libnccl.so.2", RTLD_NOW | RTLD_NOLOAD);
    if (h == nullptr) h = dlopen("libnccl.so.2", RTLD_NOW | RTLD_GLOBAL);
    if (h == nullptr) return;
    g_nccl.group_start = reinterpret_cast<decltype(g_nccl.group_start)>(dlsym(h, "ncclGroupStart"));
    g_nccl.group_end = reinterpret_cast<decltype(g_nccl.group_end)>(dlsym(h, "ncclGroupEnd"));
    g_nccl.send = reinterpret_cast<decltype(g_nccl.send)>(dlsym(h, "ncclSend"));
    g_nccl.recv = reinterpret_cast<decltype(g_nccl.recv)>(dlsym(h, "ncclRecv"));
    g_nccl.count = reinterpret_cast<decltype(g_nccl.count)>(dlsym(h, "ncclCommCount"));
    g_nccl.user_rank = reinterpret_cast<decltype(g_nccl.user_rank)>(dlsym(h, "ncclCommUserRank"));
    g_nccl.ok = g_nccl.group_start && g_nccl.group_end && g_nccl.send && g_nccl.recv &&
                g_nccl.count && g_nccl.user_rank;
}

const NcclApi *nccl()
{
    std::call_once(g_nccl_once, load_nccl);
    return g_nccl.ok ? &g_nccl : nullptr;
}

// out[q] = [rows_rank[q], cnt_expert[q*epr], ..., cnt_expert[q*epr + epr-1]]
__global__ void pack_counts_kernel(const int32_t *__restrict__ rows_rank,
                                   const int32_t *__restrict__ cnt_expert, int W, int epr,
                                   int32_t *__restrict__ out)
{
    const int n = W * (1 + epr);
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
        const int q = i / (1 + epr), c = i - q * (1 + epr);
        out[i] = c == 0 ? rows_rank[q] : cnt_expert[q * epr + c - 1];
    }
}

ep_status comm_shape(const NcclApi *api, ncclComm_t comm, int &W, int &me)
{
    if (api->count(comm, &W) != ncclSuccess || api->user_rank(comm, &me) != ncclSuccess)
        return EP_ERR_CUDA;
    return (W >= 1 && me >= 0 && me < W) ? EP_OK : EP_ERR_INVALID;
}

// Rows [off_s[q], off_s[q] + n_s[q]) of `src` go to rank q; rows from rank
// q land at [off_r[q], off_r[q] + n_r[q]) of `dst` (offsets: prefix sums of
// the counts).  The rank's own share is a device-to-device copy.
ep_status exchange_rows(ncclComm_t comm, const void *src, const int32_t *n_send,
                        const int32_t *n_recv, size_t row_bytes, void *dst, cudaStream_t s)
{
    const NcclApi *api = nccl();
    if (api == nullptr) return EP_ERR_UNSUPPORTED;
    int W = 0, me = 0;
    ep_status st = comm_shape(api, comm, W, me);
    if (st != EP_OK) return st;
    if (!n_send || !n_recv || row_bytes == 0) return EP_ERR_INVALID;
    size_t tot_s = 0, tot_r = 0;
    for (int q = 0; q < W; ++q) {
        if (n_send[q] < 0 || n_recv[q] < 0) return EP_ERR_INVALID;
        tot_s += (size_t)n_send[q];
        tot_r += (size_t)n_recv[q];
    }
    if ((tot_s && !src) || (tot_r && !dst)) return EP_ERR_INVALID;
    const char *in = static_cast<const char *>(src);
    char *out = static_cast<char *>(dst);
    if (api->group_start() != ncclSuccess) return EP_ERR_CUDA;
    size_t os = 0, orr = 0;
    ep_status res = EP_OK;
    for (int q = 0; q < W && res == EP_OK; ++q) {
        const size_t bs = (size_t)n_send[q] * row_bytes, br = (size_t)n_recv[q] * row_bytes;
        if (q == me) {
            if (bs != br) res = EP_ERR_INVALID;  // a rank's own share is the same rows
            else if (bs && cudaMemcpyAsync(out + orr, in + os, bs, cudaMemcpyDeviceToDevice, s) !=
                               cudaSuccess)
                res = EP_ERR_CUDA;
        } else {
            if (bs && api->send(in + os, bs, ncclUint8, q, comm, s) != ncclSuccess) res = EP_ERR_CUDA;
            if (br && api->recv(out + orr, br, ncclUint8, q, comm, s) != ncclSuccess) res = EP_ERR_CUDA;
        }
        os += bs;
        orr += br;
    }
    if (api->group_end() != ncclSuccess && res == EP_OK) res = EP_ERR_CUDA;
    return res;
}

}  // namespace
}  // namespace ep

using namespace ep;

extern "C" {

ep_status ep_exchange_counts(ep_nccl_comm comm, const int32_t *rows_rank,
                             const int32_t *cnt_expert, int P, int32_t *send_scratch,
                             int32_t *recv_counts, ep_stream_t stream)
{
    EP_TRACE("ep_exchange_counts");
    const NcclApi *api = nccl();
    if (api == nullptr) return EP_ERR_UNSUPPORTED;
    if (comm == nullptr || !rows_rank || !cnt_expert || !send_scratch || !recv_counts || P < 1)
        return EP_ERR_INVALID;
    ncclComm_t c = reinterpret_cast<ncclComm_t>(comm);
    int W = 0, me = 0;
    ep_status st = comm_shape(api, c, W, me);
    if (st != EP_OK) return st;
    if (P % W != 0) return EP_ERR_INVALID;
    const int epr = P / W;
    const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const int n = W * (1 + epr);
    pack_counts_kernel<<<(n + 255) / 256, 256, 0, s>>>(rows_rank, cnt_expert, W, epr,
                                                       send_scratch);
    if (cudaGetLastError() != cudaSuccess) return EP_ERR_CUDA;
    if (api->group_start() != ncclSuccess) return EP_ERR_CUDA;
    ep_status res = EP_OK;
    const size_t row = (size_t)(1 + epr);
    for (int q = 0; q < W && res == EP_OK; ++q) {
        if (api->send(send_scratch + q * row, row, ncclInt32, q, c, s) != ncclSuccess ||
            api->recv(recv_counts + q * row, row, ncclInt32, q, c, s) != ncclSuccess)
            res = EP_ERR_CUDA;
    }
    if (api->group_end() != ncclSuccess && res == EP_OK) res = EP_ERR_CUDA;
    return res;
}

ep_status ep_dispatch_exchange(ep_nccl_comm comm, const void *rows, const int32_t *send_rows,
                               const int32_t *recv_rows, size_t row_bytes, void *recv,
                               ep_stream_t stream)
{
    EP_TRACE("ep_dispatch_exchange");
    if (comm == nullptr) return EP_ERR_INVALID;
    return exchange_rows(reinterpret_cast<ncclComm_t>(comm), rows, send_rows, recv_rows,
                         row_bytes, recv, reinterpret_cast<cudaStream_t>(stream));
}

ep_status ep_combine_exchange(ep_nccl_comm comm, const void *expert_rows,
                              const int32_t *recv_rows, const int32_t *send_rows,
                              size_t row_bytes, void *back, ep_stream_t stream)
{
    EP_TRACE("ep_combine_exchange");
    if (comm == nullptr) return EP_ERR_INVALID;
    // the reverse direction: what arrived from rank q goes back to rank q
    return exchange_rows(reinterpret_cast<ncclComm_t>(comm), expert_rows, recv_rows, send_rows,
                         row_bytes, back, reinterpret_cast<cudaStream_t>(stream));
}

}  // extern "C"
