"""ctypes binding of libep_b200.so: the C-ABI calls under the same names.

Argument marshalling only: tensors become device pointers, the current torch
stream becomes the stream handle, ep_status codes become exceptions.  Every
step of the path runs in the library's CUDA kernels; there is no fallback.
"""

from __future__ import annotations

import ctypes
import os

import torch

from .build import LOAD_LIB as LIB

_lib = None

EP_OK = 0
EP_ERR_INVALID = 1
EP_ERR_UNSUPPORTED = 2
EP_ERR_CUDA = 3
EP_ERR_DEVICE = 4
EP_DEV_BAD_EXPERT = 1
EP_DEV_BAD_REPLICA = 2
EP_DEV_TIMEOUT = 4

# every symbol declared in include/ep.h and include/ep_testing.h
EXPORTS = ("ep_workspace_size", "ep_route", "ep_dispatch_layout", "ep_dispatch",
           "ep_combine", "ep_status_string", "ep_dispatch_layout_noalloc", "ep_route_layout",
           "ep_dispatch_backward", "ep_combine_backward", "ep_silu_mul", "ep_route_dispatch",
           "ep_testing_set_wait_limit", "ep_exchange_counts", "ep_dispatch_exchange",
           "ep_combine_exchange", "ep_peer_counts", "ep_peer_dispatch", "ep_peer_wait_dispatch",
           "ep_peer_experts_ready", "ep_peer_combine")
EP_DEV_OVERFLOW = 8


class EpError(RuntimeError):
    def __init__(self, fn, status):
        self.status = status
        msg = lib().ep_status_string(status).decode()
        super().__init__(f"{fn}: {msg}")


class RouteCfg(ctypes.Structure):
    _fields_ = [("num_experts", ctypes.c_int), ("n_group", ctypes.c_int),
                ("topk_group", ctypes.c_int), ("topk", ctypes.c_int),
                ("routed_scale", ctypes.c_float), ("renorm", ctypes.c_int)]


class PeerGroup(ctypes.Structure):
    """ep_peer_group: the rank-indexed tables are device addresses of arrays
    of W device pointers."""
    _fields_ = [("world", ctypes.c_int), ("rank0", ctypes.c_int), ("n_local", ctypes.c_int),
                ("P", ctypes.c_int), ("row_align", ctypes.c_int), ("cap", ctypes.c_int),
                ("recv_x", ctypes.c_void_p), ("recv_scale", ctypes.c_void_p),
                ("y", ctypes.c_void_p), ("board", ctypes.c_void_p), ("flags", ctypes.c_void_p)]


class PeerRank(ctypes.Structure):
    """ep_peer_rank: one local rank's own arrays (device addresses)."""
    _fields_ = [("x", ctypes.c_void_p), ("cnt_expert", ctypes.c_void_p),
                ("expert_off", ctypes.c_void_p), ("slot", ctypes.c_void_p),
                ("topk_w", ctypes.c_void_p), ("out", ctypes.c_void_p),
                ("dest_off", ctypes.c_void_p), ("recv_cnt", ctypes.c_void_p),
                ("recv_rows", ctypes.c_void_p), ("pair_dest", ctypes.c_void_p),
                ("dev_status", ctypes.c_void_p),
                ("T", ctypes.c_int), ("reserved", ctypes.c_int)]


def lib() -> ctypes.CDLL:
    """The loaded library; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB):
            raise ImportError(
                f"libep_b200.so not found at {LIB}; build it with "
                "`python -m combine_ep_route_02_b200.build` (nvcc, sm_100a)")
        L = ctypes.CDLL(LIB)
        P, I, F, Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
        L.ep_workspace_size.argtypes = [I, I, I, I]
        L.ep_workspace_size.restype = Z
        L.ep_route.argtypes = [P, P, I, RouteCfg, P, P, P]
        L.ep_route.restype = I
        L.ep_dispatch_layout.argtypes = [P, I, I, I, I, I, P, P, I, I,
                                         P, P, P, P, P, P, P, P, P, P, P]
        L.ep_dispatch_layout.restype = I
        L.ep_dispatch.argtypes = [P, I, I, I, I, P, I, P, P, I, P, P]
        L.ep_dispatch.restype = I
        L.ep_combine.argtypes = [P, P, P, I, I, I, I, P, I, P, P]
        L.ep_combine.restype = I
        L.ep_dispatch_layout_noalloc.argtypes = [P, I, I, I, I, I, P, P, I,
                                                 P, P, P, P, P, P, P, P, P, P]
        L.ep_dispatch_layout_noalloc.restype = I
        L.ep_route_layout.argtypes = [P, P, I, RouteCfg, I, I, P, P, I, I,
                                      P, P, P, P, P, P, P, P, P, P, P, P, P]
        L.ep_route_layout.restype = I
        L.ep_dispatch_backward.argtypes = [P, P, I, I, I, I, P, I, P, P]
        L.ep_dispatch_backward.restype = I
        L.ep_combine_backward.argtypes = [P, P, P, P, I, I, I, I, P, P, I, P, P]
        L.ep_combine_backward.restype = I
        L.ep_silu_mul.argtypes = [P, I, I, P, P, I, I, P, P, I, P]
        L.ep_silu_mul.restype = I
        L.ep_route_dispatch.argtypes = [P, P, I, RouteCfg, I, I, P, P, I, I, P, I, I, I, P, P,
                                        P, P, P, P, P, P, P, P, P, P, P, I, P, P]
        L.ep_route_dispatch.restype = I
        L.ep_testing_set_wait_limit.argtypes = [ctypes.c_longlong]
        L.ep_testing_set_wait_limit.restype = I
        L.ep_exchange_counts.argtypes = [P, P, P, I, P, P, P]
        L.ep_exchange_counts.restype = I
        L.ep_dispatch_exchange.argtypes = [P, P, P, P, Z, P, P]
        L.ep_dispatch_exchange.restype = I
        L.ep_combine_exchange.argtypes = [P, P, P, P, Z, P, P]
        L.ep_combine_exchange.restype = I
        G, RP = PeerGroup, ctypes.c_void_p
        L.ep_peer_counts.argtypes = [G, RP, I, I, P]
        L.ep_peer_counts.restype = I
        L.ep_peer_dispatch.argtypes = [G, RP, I, I, I, P]
        L.ep_peer_dispatch.restype = I
        L.ep_peer_wait_dispatch.argtypes = [G, RP, P]
        L.ep_peer_wait_dispatch.restype = I
        L.ep_peer_experts_ready.argtypes = [G, P]
        L.ep_peer_experts_ready.restype = I
        L.ep_peer_combine.argtypes = [G, RP, I, I, I, P]
        L.ep_peer_combine.restype = I
        L.ep_status_string.argtypes = [I]
        L.ep_status_string.restype = ctypes.c_char_p
        _lib = L
    return _lib


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(fn, st):
    if st != EP_OK:
        raise EpError(fn, st)


def ep_workspace_size(T: int, k: int, P: int, R: int) -> int:
    return int(lib().ep_workspace_size(T, k, P, R))


def ep_route(logits, bias, T, cfg: RouteCfg, topk_idx, topk_w, stream=None):
    _check("ep_route", lib().ep_route(_ptr(logits), _ptr(bias), T, cfg, _ptr(topk_idx),
                                      _ptr(topk_w), _stream(stream)))


def ep_dispatch_layout(topk_idx, T, k, E, P, R, phys_of, n_rep, max_rep, cnt_expert,
                       expert_off, rows_rank, rank_off, tok_rank, in_rank, slot, src,
                       workspace, dev_status, stream=None, *, row_align=1):
    """row_align > 1: each expert's rows start on a multiple of row_align and
    src needs T*k + P*(row_align-1) entries."""
    _check("ep_dispatch_layout", lib().ep_dispatch_layout(
        _ptr(topk_idx), T, k, E, P, R, _ptr(phys_of), _ptr(n_rep), max_rep, row_align,
        _ptr(cnt_expert), _ptr(expert_off), _ptr(rows_rank), _ptr(rank_off), _ptr(tok_rank),
        _ptr(in_rank), _ptr(slot), _ptr(src), _ptr(workspace), _ptr(dev_status),
        _stream(stream)))


def ep_dispatch(x, T, H, k, slot, fp8, recv_x, recv_scale, num_sms=0, dev_status=None,
                stream=None, *, recv_rows=0):
    """recv_rows: rows of recv_x (0 = T*k)."""
    _check("ep_dispatch", lib().ep_dispatch(_ptr(x), T, H, k, recv_rows, _ptr(slot),
                                            int(bool(fp8)), _ptr(recv_x), _ptr(recv_scale),
                                            num_sms, _ptr(dev_status), _stream(stream)))


def ep_combine(y, slot, topk_w, T, H, k, out, num_sms=0, dev_status=None, stream=None, *,
               recv_rows=0):
    """recv_rows: rows of y (0 = T*k)."""
    _check("ep_combine", lib().ep_combine(_ptr(y), _ptr(slot), _ptr(topk_w), T, H, k, recv_rows,
                                          _ptr(out), num_sms, _ptr(dev_status),
                                          _stream(stream)))


def ep_dispatch_layout_noalloc(topk_idx, T, k, E, P, R, phys_of, n_rep, max_rep, cnt_expert,
                               expert_off, rows_rank, rank_off, tok_rank, in_rank, slot, src,
                               dev_status, stream=None):
    """ep_dispatch_layout with the library's fixed device scratch instead of a
    caller-provided workspace (for callers that cannot allocate device memory)."""
    _check("ep_dispatch_layout_noalloc", lib().ep_dispatch_layout_noalloc(
        _ptr(topk_idx), T, k, E, P, R, _ptr(phys_of), _ptr(n_rep), max_rep,
        _ptr(cnt_expert), _ptr(expert_off), _ptr(rows_rank), _ptr(rank_off), _ptr(tok_rank),
        _ptr(in_rank), _ptr(slot), _ptr(src), _ptr(dev_status), _stream(stream)))


def ep_route_layout(logits, bias, T, cfg: RouteCfg, P, R, phys_of, n_rep, max_rep, topk_idx,
                    topk_w, cnt_expert, expert_off, rows_rank, rank_off, tok_rank, in_rank, slot,
                    src, workspace, dev_status, stream=None, *, row_align=1):
    """ep_route followed by ep_dispatch_layout (one kernel for small batches)."""
    _check("ep_route_layout", lib().ep_route_layout(
        _ptr(logits), _ptr(bias), T, cfg, P, R, _ptr(phys_of), _ptr(n_rep), max_rep, row_align,
        _ptr(topk_idx), _ptr(topk_w), _ptr(cnt_expert), _ptr(expert_off), _ptr(rows_rank),
        _ptr(rank_off), _ptr(tok_rank), _ptr(in_rank), _ptr(slot), _ptr(src), _ptr(workspace),
        _ptr(dev_status), _stream(stream)))


def ep_route_dispatch(logits, bias, T, cfg: RouteCfg, P, R, phys_of, n_rep, max_rep, x, H, fp8,
                      recv_x, recv_scale, topk_idx, topk_w, cnt_expert, expert_off, rows_rank,
                      rank_off, tok_rank, in_rank, slot, src, workspace, dev_status, stream=None,
                      *, row_align=1, recv_rows=0, num_sms=0):
    """ep_route_layout followed by ep_dispatch (one kernel for small batches)."""
    _check("ep_route_dispatch", lib().ep_route_dispatch(
        _ptr(logits), _ptr(bias), T, cfg, P, R, _ptr(phys_of), _ptr(n_rep), max_rep, row_align,
        _ptr(x), H, int(bool(fp8)), recv_rows, _ptr(recv_x), _ptr(recv_scale), _ptr(topk_idx),
        _ptr(topk_w), _ptr(cnt_expert), _ptr(expert_off), _ptr(rows_rank), _ptr(rank_off),
        _ptr(tok_rank), _ptr(in_rank), _ptr(slot), _ptr(src), _ptr(workspace), num_sms,
        _ptr(dev_status), _stream(stream)))


def ep_testing_set_wait_limit(polls: int):
    """Failure-detection tests only: polls of every bounded device wait in
    later launches (0 = give up at once, negative = the default)."""
    _check("ep_testing_set_wait_limit", lib().ep_testing_set_wait_limit(int(polls)))


def _host_i32(counts):
    """host int32 array (kept alive by the caller) of a list of counts"""
    import numpy as np
    return np.ascontiguousarray(np.asarray(counts, dtype=np.int32))


def ep_exchange_counts(comm: int, rows_rank, cnt_expert, P, send_scratch, recv_counts,
                       stream=None):
    """comm: the ncclComm_t (an integer address) of a NCCL process group."""
    _check("ep_exchange_counts", lib().ep_exchange_counts(
        comm, _ptr(rows_rank), _ptr(cnt_expert), P, _ptr(send_scratch), _ptr(recv_counts),
        _stream(stream)))


def ep_dispatch_exchange(comm: int, rows, send_rows, recv_rows, row_bytes: int, recv,
                         stream=None):
    """send_rows / recv_rows: host counts per rank (lists or arrays)."""
    s, r = _host_i32(send_rows), _host_i32(recv_rows)
    _check("ep_dispatch_exchange", lib().ep_dispatch_exchange(
        comm, _ptr(rows), s.ctypes.data, r.ctypes.data, row_bytes, _ptr(recv), _stream(stream)))


def ep_combine_exchange(comm: int, expert_rows, recv_rows, send_rows, row_bytes: int, back,
                        stream=None):
    s, r = _host_i32(send_rows), _host_i32(recv_rows)
    _check("ep_combine_exchange", lib().ep_combine_exchange(
        comm, _ptr(expert_rows), r.ctypes.data, s.ctypes.data, row_bytes, _ptr(back),
        _stream(stream)))


def ep_peer_counts(group: PeerGroup, ranks_dev, k, max_T, stream=None):
    """ranks_dev: device buffer holding n_local PeerRank structs."""
    _check("ep_peer_counts", lib().ep_peer_counts(group, _ptr(ranks_dev), k, max_T,
                                                  _stream(stream)))


def ep_peer_dispatch(group: PeerGroup, ranks_dev, H, k, max_T, stream=None):
    _check("ep_peer_dispatch", lib().ep_peer_dispatch(group, _ptr(ranks_dev), H, k, max_T,
                                                      _stream(stream)))


def ep_peer_wait_dispatch(group: PeerGroup, ranks_dev, stream=None):
    _check("ep_peer_wait_dispatch", lib().ep_peer_wait_dispatch(group, _ptr(ranks_dev),
                                                                _stream(stream)))


def ep_peer_experts_ready(group: PeerGroup, stream=None):
    _check("ep_peer_experts_ready", lib().ep_peer_experts_ready(group, _stream(stream)))


def ep_peer_combine(group: PeerGroup, ranks_dev, H, k, max_T, stream=None):
    _check("ep_peer_combine", lib().ep_peer_combine(group, _ptr(ranks_dev), H, k, max_T,
                                                    _stream(stream)))


def ep_dispatch_backward(grad_recv, slot, T, H, k, grad_x, num_sms=0, dev_status=None,
                         stream=None, *, recv_rows=0):
    _check("ep_dispatch_backward", lib().ep_dispatch_backward(
        _ptr(grad_recv), _ptr(slot), T, H, k, recv_rows, _ptr(grad_x), num_sms,
        _ptr(dev_status), _stream(stream)))


def ep_combine_backward(grad_out, y, slot, topk_w, T, H, k, grad_y, grad_w, num_sms=0,
                        dev_status=None, stream=None, *, recv_rows=0):
    _check("ep_combine_backward", lib().ep_combine_backward(
        _ptr(grad_out), _ptr(y), _ptr(slot), _ptr(topk_w), T, H, k, recv_rows, _ptr(grad_y),
        _ptr(grad_w), num_sms, _ptr(dev_status), _stream(stream)))


def ep_silu_mul(gate_up, n_rows, I, expert_off, cnt_expert, P, fp8, act, act_scale, num_sms=0,
                stream=None):
    """silu(gate) * up of the rows [expert_off[p], expert_off[p] + cnt_expert[p])
    (every row when both are None), e4m3 + 1x128 scales when fp8, else bf16."""
    _check("ep_silu_mul", lib().ep_silu_mul(
        _ptr(gate_up), n_rows, I, _ptr(expert_off), _ptr(cnt_expert), P, int(bool(fp8)),
        _ptr(act), _ptr(act_scale), num_sms, _stream(stream)))
