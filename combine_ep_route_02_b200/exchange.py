"""Expert parallelism across processes: the exchange between each rank's
rank-major receive rows and the ranks that own the experts.

On one GPU the expert-parallel ranks are logical: rank r's rows are the range
[rank_off[r], rank_off[r+1]) of one buffer.  Across processes (one per GPU),
rank r of a process group owns physical experts [r*P/R, (r+1)*P/R), and that
range of every rank's receive buffer has to reach it: the dispatch
all-to-all, and in reverse the combine all-to-all, of the Perplexity blog's
section "Expert Parallelism".  The local kernels are unchanged: the layout
already writes each destination's rows contiguously, so each direction is one
all-to-all-v of whole rows, and the combine runs locally on the rows that
come back in their original order.

The split sizes are the layout's ``rows_rank``; they are needed as host
integers, so building an ``ExchangePlan`` copies the counts to the host once
per layout (the handle of the DeepEP V2 summary is reused for the combine
direction).  Rows travel as raw bytes, so e4m3 codes, fp32 scales and bf16
rows use the same calls.

In a NCCL process group every step runs in the C library on the group's own
communicator (``ep_exchange_counts``, ``ep_dispatch_exchange``,
``ep_combine_exchange``: grouped NCCL sends and receives, over NVLink between
GPUs); this module only marshals arguments.  Other backends (gloo, CPU
tensors) take torch.distributed's all-to-all with the same split sizes.
"""

from __future__ import annotations

from dataclasses import dataclass
from typing import List, Optional

import torch
import torch.distributed as dist


@dataclass
class ExchangePlan:
    """Split sizes of one layout's exchange, seen from this rank.

    send_splits[r]  rows this rank sends to rank r (its rows_rank[r])
    recv_splits[s]  rows this rank receives from rank s
    recv_cnt[s][e]  pairs from rank s for this rank's local expert e (the
                    per-expert counts a grouped GEMM needs, per source)
    """
    send_splits: List[int]
    recv_splits: List[int]
    recv_cnt: torch.Tensor  # int64 [R, P/R], on the host
    rank: int
    world: int


def _host_ints(t) -> torch.Tensor:
    return torch.as_tensor(t).detach().to("cpu", torch.int64).reshape(-1)


_COMM_READY = set()


def _nccl_comm(group) -> Optional[int]:
    """The ncclComm_t (as an integer) behind a NCCL process group on the
    current device, or None for another backend."""
    if dist.get_backend(group) != "nccl":
        return None
    pg = group if group is not None else dist.distributed_c10d._get_default_group()
    dev = torch.device("cuda", torch.cuda.current_device())
    key = (id(pg), dev.index)
    if key not in _COMM_READY:
        # the group creates its communicator lazily, at its first collective
        dist.all_reduce(torch.zeros(1, device=dev), group=group)
        torch.cuda.synchronize(dev)
        _COMM_READY.add(key)
    return int(pg._get_backend(dev)._comm_ptr())


def exchange_plan(rows_rank, cnt_expert, group=None) -> ExchangePlan:
    """Exchanges the per-destination row counts and per-expert pair counts.

    rows_rank   [R] rows of this rank's receive buffer for each rank (R must
                equal the group's size)
    cnt_expert  [P] pairs of this rank per physical expert (P % R == 0)
    """
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    rr = _host_ints(rows_rank)
    ce = _host_ints(cnt_expert)
    if rr.numel() != world:
        raise ValueError(f"rows_rank has {rr.numel()} ranks, the group has {world}")
    if ce.numel() % world:
        raise ValueError("the number of physical experts must be a multiple of the group size")
    epr = ce.numel() // world
    comm = _nccl_comm(group)
    if comm is not None:
        # the counts' all-to-all in the library, on the group's communicator;
        # then the one device-to-host read of the layout
        from . import _binding as B
        dev = torch.device("cuda", torch.cuda.current_device())
        rr_d = torch.as_tensor(rows_rank).to(dev, torch.int32).contiguous()
        ce_d = torch.as_tensor(cnt_expert).to(dev, torch.int32).contiguous()
        send = torch.empty((world, 1 + epr), dtype=torch.int32, device=dev)
        recv = torch.empty_like(send)
        B.ep_exchange_counts(comm, rr_d, ce_d, ce.numel(), send, recv)
        recv = recv.cpu().to(torch.int64)
    else:
        # one all-to-all of [rows, count of each local expert] per destination
        send = torch.cat([rr.view(world, 1), ce.view(world, epr)], dim=1).contiguous()
        recv = torch.empty_like(send)
        dist.all_to_all_single(recv, send, group=group)
    return ExchangePlan(send_splits=rr.tolist(), recv_splits=recv[:, 0].tolist(),
                        recv_cnt=recv[:, 1:].clone(), rank=rank, world=world)


def _row_bytes(t: torch.Tensor) -> int:
    n = t.element_size()
    for d in t.shape[1:]:
        n *= d
    return n


def _as_bytes(rows: torch.Tensor, writable: bool = False) -> torch.Tensor:
    """[N, ...] rows as a uint8 [N, row_bytes] view (a contiguous copy for a
    read-only source; a destination must already be contiguous)."""
    if writable and not rows.is_contiguous():
        raise ValueError("the exchange's output buffer must be contiguous")
    r = rows.contiguous()
    return r.view(torch.uint8).reshape(r.shape[0], _row_bytes(r))


def dispatch_exchange(send_rows: torch.Tensor, plan: ExchangePlan, group=None,
                      out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Sends rows [rank_off[r], rank_off[r+1]) of this rank's receive buffer
    to rank r; returns the rows this rank receives, grouped by source rank
    (and within a source by expert, as the source's layout ordered them).

    send_rows  [N, ...] the receive buffer (or its scales); its first
               sum(send_splits) rows are sent
    out        optional [sum(recv_splits), ...] contiguous result buffer
    """
    n_send, n_recv = sum(plan.send_splits), sum(plan.recv_splits)
    if out is None:
        out = torch.empty((n_recv,) + tuple(send_rows.shape[1:]), dtype=send_rows.dtype,
                          device=send_rows.device)
    dst, src = _as_bytes(out[:n_recv], True), _as_bytes(send_rows[:n_send])
    comm = _nccl_comm(group)
    if comm is not None:
        from . import _binding as B
        B.ep_dispatch_exchange(comm, src, plan.send_splits, plan.recv_splits,
                               _row_bytes(send_rows), dst)
    else:
        dist.all_to_all_single(dst, src, output_split_sizes=plan.recv_splits,
                               input_split_sizes=plan.send_splits, group=group)
    return out


def combine_exchange(expert_rows: torch.Tensor, plan: ExchangePlan, group=None,
                     out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """The reverse of dispatch_exchange: expert outputs for the received rows
    (in received order) go back to their source ranks; returns this rank's
    rows in its own receive-row order, ready for the local combine.

    expert_rows  [sum(recv_splits), ...] outputs of this rank's experts
    out          optional [sum(send_splits), ...] contiguous result buffer
    """
    n_send, n_recv = sum(plan.send_splits), sum(plan.recv_splits)
    if out is None:
        out = torch.empty((n_send,) + tuple(expert_rows.shape[1:]), dtype=expert_rows.dtype,
                          device=expert_rows.device)
    dst, src = _as_bytes(out[:n_send], True), _as_bytes(expert_rows[:n_recv])
    comm = _nccl_comm(group)
    if comm is not None:
        from . import _binding as B
        B.ep_combine_exchange(comm, src, plan.recv_splits, plan.send_splits,
                              _row_bytes(expert_rows), dst)
    else:
        dist.all_to_all_single(dst, src, output_split_sizes=plan.send_splits,
                               input_split_sizes=plan.recv_splits, group=group)
    return out
