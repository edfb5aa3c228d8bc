"""The MoE routing -> layout -> dispatch -> combine path over caller-owned
device buffers.

``EpPath`` allocates every buffer once with torch (device memory is the only
thing torch provides here) and then issues the four C-ABI calls on one
stream.  No call synchronises the host; per-expert counts stay on the device
until the caller copies them (the DeepEP V2 handle's
num_recv_tokens_per_expert_list).
"""

from __future__ import annotations

from typing import Optional

import torch

from . import _binding as B


class EpPath:
    """Buffers and calls for one (T, H, routing, ranks) shape.

    The receive buffers have T*k rows: rank r's rows are
    ``recv_x[rank_off[r]:rank_off[r+1]]`` and expert p's rows are
    ``recv_x[expert_off[p]:expert_off[p+1]]``.
    """

    def __init__(self, T: int, H: int, num_experts: int, n_group: int, topk_group: int,
                 topk: int, routed_scale: float, renorm: bool, R: int, fp8: bool,
                 phys_of: Optional[torch.Tensor] = None, n_rep: Optional[torch.Tensor] = None,
                 device="cuda", num_sms: int = 0):
        dev = torch.device(device)
        self.T, self.H, self.k, self.E, self.R = T, H, topk, num_experts, R
        self.fp8 = bool(fp8)
        self.num_sms = num_sms
        self.cfg = B.RouteCfg(num_experts, n_group, topk_group, topk, float(routed_scale),
                              int(bool(renorm)))
        if phys_of is not None:
            self.phys_of = phys_of.to(dev, torch.int32).contiguous()
            self.n_rep = n_rep.to(dev, torch.int32).contiguous()
            self.max_rep = int(self.phys_of.shape[1])
            self.P = int(self.phys_of.max().item()) + 1
        else:
            self.phys_of = self.n_rep = None
            self.max_rep = 0
            self.P = num_experts
        P, k = self.P, topk
        i32 = dict(device=dev, dtype=torch.int32)
        self.topk_idx = torch.empty((T, k), **i32)
        self.topk_w = torch.empty((T, k), device=dev, dtype=torch.float32)
        self.cnt_expert = torch.empty(P, **i32)
        self.expert_off = torch.empty(P + 1, **i32)
        self.rows_rank = torch.empty(R, **i32)
        self.rank_off = torch.empty(R + 1, **i32)
        self.tok_rank = torch.empty(R, **i32)
        self.in_rank = torch.empty((T, R), device=dev, dtype=torch.uint8)
        self.slot = torch.empty((T, k), **i32)
        self.src = torch.empty(T * k, **i32)
        self.dev_status = torch.zeros(1, **i32)    # layout (cleared by each layout call)
        self.copy_status = torch.zeros(1, **i32)   # dispatch / combine (sticky)
        ws = B.ep_workspace_size(T, k, P, R)
        self.workspace = torch.empty(max(ws, 256), device=dev, dtype=torch.uint8)
        if self.fp8:
            self.recv_x = torch.empty((T * k, H), device=dev, dtype=torch.float8_e4m3fn)
            self.recv_scale = torch.empty((T * k, H // 128), device=dev, dtype=torch.float32)
        else:
            self.recv_x = torch.empty((T * k, H), device=dev, dtype=torch.bfloat16)
            self.recv_scale = None
        self.out = torch.empty((T, H), device=dev, dtype=torch.bfloat16)

    # the four steps -------------------------------------------------------
    def route(self, logits: torch.Tensor, bias: Optional[torch.Tensor], stream=None):
        B.ep_route(logits, bias, self.T, self.cfg, self.topk_idx, self.topk_w, stream)

    def layout(self, stream=None):
        B.ep_dispatch_layout(self.topk_idx, self.T, self.k, self.E, self.P, self.R,
                             self.phys_of, self.n_rep, self.max_rep, self.cnt_expert,
                             self.expert_off, self.rows_rank, self.rank_off, self.tok_rank,
                             self.in_rank, self.slot, self.src, self.workspace,
                             self.dev_status, stream)

    def dispatch(self, x: torch.Tensor, stream=None):
        B.ep_dispatch(x, self.T, self.H, self.k, self.slot, self.fp8, self.recv_x,
                      self.recv_scale, self.num_sms, self.copy_status, stream)

    def combine(self, y: torch.Tensor, stream=None):
        B.ep_combine(y, self.slot, self.topk_w, self.T, self.H, self.k, self.out,
                     self.num_sms, self.copy_status, stream)

    def step(self, x, logits, bias, y, stream=None):
        """route, layout, dispatch, then combine of the expert outputs y."""
        self.route(logits, bias, stream)
        self.layout(stream)
        self.dispatch(x, stream)
        self.combine(y, stream)
        return self.out

    def kernels_per_step(self) -> int:
        """Kernels one step launches: route, layout (count + slot, plus a
        column scan above 64 tiles), dispatch, combine.  Mirrors the tiling
        rule of the layout (64..512 tokens per tile, at most 64 tiles while
        tiles can grow, capped by the slot kernel's shared memory)."""
        if self.T == 0:
            return 1
        tt = max(64, min(512, -(-self.T // 64)))
        hw = 32
        while hw > 1 and hw * self.P > 32768:
            hw //= 2
        cap = max(32, ((51200 - (2 * self.P + 1) - hw * self.P) // self.k) // 32 * 32)
        tt = min(tt, cap)
        n_tiles = -(-self.T // tt)
        return 1 + (2 if n_tiles <= 64 else 3) + 1 + 1

    def check_status(self):
        """Reads the device status words (synchronises); raises on bad data
        or a timed-out copy."""
        st = int(self.dev_status.item()) | int(self.copy_status.item())
        if st:
            raise B.EpError("ep path (device status %#x)" % st, B.EP_ERR_DEVICE)
        return st
