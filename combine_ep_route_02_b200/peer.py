"""Expert parallelism over peer memory: buffers and calls around the
library's ep_peer_* entry points (argument marshalling only).

``EpPeerRanks`` keeps the buffers of the ranks one process serves on its
GPU and issues the step: counts, dispatch, wait, (experts), ready, combine.
Its receive buffers are addressed through rank-indexed device tables:

* ``EpPeerRanks.local(...)`` puts all W ranks on this GPU (each its own
  allocations; the kernels cover every rank in one launch), which is how a
  one-GPU run exercises the protocol;
* ``EpPeerRanks.from_process_group(...)`` serves one rank per process and
  maps the other ranks' buffers with CUDA IPC (torch's storage sharing),
  exchanged over the process group; on one node, over NVLink.
"""

from __future__ import annotations

import ctypes
from typing import Callable, List, Optional

import numpy as np
import torch

from . import _binding as B


def _ptr_table(tensors, device) -> torch.Tensor:
    return torch.tensor([t.data_ptr() for t in tensors], dtype=torch.int64, device=device)


class EpPeerRanks:
    """Buffers of the ranks ``rank0 .. rank0 + n_local - 1`` of a W-rank
    expert-parallel group, and the peer step over them.

    paths   one ``EpPath`` per local rank (R = W) laying out its tokens
    cap     rows of every rank's receive buffers
    """

    def __init__(self, world: int, rank0: int, paths, H: int, cap: int, row_align: int,
                 recv_x, recv_scale, y, board, flags, device="cuda"):
        dev = torch.device(device)
        self.world, self.rank0, self.paths, self.H, self.cap = world, rank0, paths, H, cap
        self.n_local = len(paths)
        self.k = paths[0].k
        self.P = paths[0].P
        self.row_align = row_align
        # own-rank buffers (index = rank - rank0) and the rank-indexed tables
        self.recv_x, self.recv_scale, self.y = recv_x, recv_scale, y
        self.board, self.flags = board, flags
        self._keep = []
        P, W = self.P, world
        epr = P // W
        i32 = dict(dtype=torch.int32, device=dev)
        self.dest_off = [torch.empty(P, **i32) for _ in paths]
        self.recv_cnt = [torch.empty((epr, W), **i32) for _ in paths]
        self.recv_rows = [torch.empty(1, **i32) for _ in paths]
        # (rank, row) of every pair, written by the counts step
        self.pair_dest = [torch.empty((p.T, p.k, 2), **i32) for p in paths]
        self.status = [torch.zeros(1, **i32) for _ in paths]

    def _tables(self, recv_x_all, recv_scale_all, y_all, board_all, flags_all, dev):
        self.t_recv_x = _ptr_table(recv_x_all, dev)
        self.t_recv_scale = _ptr_table(recv_scale_all, dev)
        self.t_y = _ptr_table(y_all, dev)
        self.t_board = _ptr_table(board_all, dev)
        self.t_flags = _ptr_table(flags_all, dev)
        self.group = B.PeerGroup(self.world, self.rank0, self.n_local, self.P, self.row_align,
                                 self.cap, self.t_recv_x.data_ptr(), self.t_recv_scale.data_ptr(),
                                 self.t_y.data_ptr(), self.t_board.data_ptr(),
                                 self.t_flags.data_ptr())

    def set_inputs(self, xs, outs):
        """Per local rank: its tokens x (bf16 [T, H]) and the combine output
        buffer (bf16 [T, H]); builds the device array of ep_peer_rank."""
        arr = (B.PeerRank * self.n_local)()
        for i, p in enumerate(self.paths):
            arr[i] = B.PeerRank(xs[i].data_ptr(), p.cnt_expert.data_ptr(),
                                p.expert_off.data_ptr(), p.slot.data_ptr(),
                                p.topk_w.data_ptr(), outs[i].data_ptr(),
                                self.dest_off[i].data_ptr(), self.recv_cnt[i].data_ptr(),
                                self.recv_rows[i].data_ptr(), self.pair_dest[i].data_ptr(),
                                self.status[i].data_ptr(),
                                p.T, 0)
        raw = np.frombuffer(bytes(arr), dtype=np.uint8)
        self.ranks_dev = torch.from_numpy(raw.copy()).to(self.t_flags.device)
        self._keep = [xs, outs]
        self.max_T = max(p.T for p in self.paths)

    # the step ---------------------------------------------------------
    def counts(self, stream=None):
        B.ep_peer_counts(self.group, self.ranks_dev, self.k, self.max_T, stream)

    def dispatch(self, stream=None):
        B.ep_peer_dispatch(self.group, self.ranks_dev, self.H, self.k, self.max_T, stream)

    def wait_dispatch(self, stream=None):
        B.ep_peer_wait_dispatch(self.group, self.ranks_dev, stream)

    def experts_ready(self, stream=None):
        B.ep_peer_experts_ready(self.group, stream)

    def combine(self, stream=None):
        B.ep_peer_combine(self.group, self.ranks_dev, self.H, self.k, self.max_T, stream)

    def step(self, experts: Callable[[int, torch.Tensor, torch.Tensor, torch.Tensor], None],
             stream=None):
        """counts, dispatch, wait, experts(i, recv_x, recv_scale, y) for each
        local rank i, ready, combine; the layouts must be current."""
        self.counts(stream)
        self.dispatch(stream)
        self.wait_dispatch(stream)
        for i in range(self.n_local):
            experts(i, self.recv_x[i], self.recv_scale[i], self.y[i])
        self.experts_ready(stream)
        self.combine(stream)

    def check_status(self) -> List[int]:
        return [int(s.item()) for s in self.status]

    # construction -----------------------------------------------------
    @staticmethod
    def capacity(total_pairs: int, P: int, world: int, row_align: int) -> int:
        """rows any rank can receive: every source's pairs plus the padding
        of its experts"""
        return total_pairs + (P // world) * (row_align - 1)

    @classmethod
    def local(cls, paths, H: int, row_align: int = 1, device="cuda"):
        """All W = len(paths) ranks on this GPU."""
        dev = torch.device(device)
        W = len(paths)
        P = paths[0].P
        cap = cls.capacity(sum(p.T * p.k for p in paths), P, W, row_align)
        rx = [torch.empty((cap, H), dtype=torch.uint8, device=dev) for _ in range(W)]
        rs = [torch.empty((cap, H // 128), dtype=torch.float32, device=dev) for _ in range(W)]
        y = [torch.empty((cap, H), dtype=torch.bfloat16, device=dev) for _ in range(W)]
        board = [torch.zeros((W, P), dtype=torch.int32, device=dev) for _ in range(W)]
        flags = [torch.zeros(8, dtype=torch.int32, device=dev) for _ in range(W)]
        self = cls(W, 0, paths, H, cap, row_align, rx, rs, y, board, flags, device)
        self._tables(rx, rs, y, board, flags, dev)
        return self

    @classmethod
    def from_process_group(cls, path, H: int, cap: int, row_align: int = 1, group=None):
        """One rank per process (rank = the group rank, world = its size);
        the other ranks' buffers are mapped with CUDA IPC.  Every rank must
        pass the same cap and row_align."""
        import torch.distributed as dist
        W, me = dist.get_world_size(group), dist.get_rank(group)
        dev = torch.device("cuda", torch.cuda.current_device())
        P = path.P
        own = dict(recv_x=torch.empty((cap, H), dtype=torch.uint8, device=dev),
                   recv_scale=torch.empty((cap, H // 128), dtype=torch.float32, device=dev),
                   y=torch.empty((cap, H), dtype=torch.bfloat16, device=dev),
                   board=torch.zeros((W, P), dtype=torch.int32, device=dev),
                   flags=torch.zeros(8, dtype=torch.int32, device=dev))
        torch.cuda.synchronize(dev)
        # every rank's IPC handles of the five buffers
        from torch.multiprocessing.reductions import reduce_tensor
        mine = {n: reduce_tensor(t) for n, t in own.items()}
        allh = [None] * W
        dist.all_gather_object(allh, mine, group=group)
        tables = {}
        for n in own:
            col = []
            for q in range(W):
                if q == me:
                    col.append(own[n])
                else:
                    fn, args = allh[q][n]
                    col.append(fn(*args))
            tables[n] = col
        self = cls(W, me, [path], H, cap, row_align, [own["recv_x"]], [own["recv_scale"]],
                   [own["y"]], [own["board"]], [own["flags"]], dev)
        self._peer_views = tables
        self._tables(tables["recv_x"], tables["recv_scale"], tables["y"], tables["board"],
                     tables["flags"], dev)
        dist.barrier(group=group)
        return self
