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

    The receive buffers have ``n_recv`` rows: T*k, plus P*(row_align-1) when
    each expert's rows start on a multiple of ``row_align`` (the GEMM layout).
    Rank r's rows are ``recv_x[rank_off[r]:rank_off[r+1]]`` and expert p's
    pairs are ``recv_x[expert_off[p]:expert_off[p] + cnt_expert[p]]``.
    """

    def __init__(self, T: int, H: int, num_experts: int, n_group: int, topk_group: int,
                 topk: int, routed_scale: float, renorm: bool, R: int, fp8: bool,
                 phys_of: Optional[torch.Tensor] = None, n_rep: Optional[torch.Tensor] = None,
                 device="cuda", num_sms: int = 0, row_align: int = 1):
        dev = torch.device(device)
        self.T, self.H, self.k, self.E, self.R = T, H, topk, num_experts, R
        self.row_align = int(row_align)
        self.fp8 = bool(fp8)
        self.num_sms = num_sms          # SMs for dispatch and combine (0 = all)
        self.dispatch_sms = num_sms
        self.combine_sms = num_sms
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
        self.n_recv = T * k + P * (self.row_align - 1)
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
        self.src = torch.empty(self.n_recv, **i32)
        self.dev_status = torch.zeros(1, **i32)    # layout (cleared by each layout call)
        self.copy_status = torch.zeros(1, **i32)   # dispatch / combine (sticky)
        ws = B.ep_workspace_size(T, k, P, R)
        # zeroed once: ep_route_dispatch keeps its counters there
        self.workspace = torch.zeros(max(ws, 256), device=dev, dtype=torch.uint8)
        n = self.n_recv
        if self.fp8:
            self.recv_x = torch.empty((n, H), device=dev, dtype=torch.float8_e4m3fn)
            self.recv_scale = torch.empty((n, H // 128), device=dev, dtype=torch.float32)
        else:
            self.recv_x = torch.empty((n, H), device=dev, dtype=torch.bfloat16)
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
                             self.dev_status, stream, row_align=self.row_align)

    def route_layout(self, logits: torch.Tensor, bias: Optional[torch.Tensor], stream=None):
        """route then layout in one call (one kernel for small batches)"""
        B.ep_route_layout(logits, bias, self.T, self.cfg, self.P, self.R, self.phys_of,
                          self.n_rep, self.max_rep, self.topk_idx, self.topk_w,
                          self.cnt_expert, self.expert_off, self.rows_rank, self.rank_off,
                          self.tok_rank, self.in_rank, self.slot, self.src, self.workspace,
                          self.dev_status, stream, row_align=self.row_align)

    def route_dispatch(self, logits: torch.Tensor, bias: Optional[torch.Tensor], x: torch.Tensor,
                       stream=None):
        """route, layout and dispatch in one call (one kernel for small
        batches); the same outputs as route_layout then dispatch.  The one
        dev_status word of the call lands in ``dev_status``."""
        B.ep_route_dispatch(logits, bias, self.T, self.cfg, self.P, self.R, self.phys_of,
                            self.n_rep, self.max_rep, x, self.H, self.fp8, self.recv_x,
                            self.recv_scale, self.topk_idx, self.topk_w, self.cnt_expert,
                            self.expert_off, self.rows_rank, self.rank_off, self.tok_rank,
                            self.in_rank, self.slot, self.src, self.workspace, self.dev_status,
                            stream, row_align=self.row_align, recv_rows=self.n_recv,
                            num_sms=self.dispatch_sms)

    def dispatch(self, x: torch.Tensor, stream=None):
        B.ep_dispatch(x, self.T, self.H, self.k, self.slot, self.fp8, self.recv_x,
                      self.recv_scale, self.dispatch_sms, self.copy_status, stream,
                      recv_rows=self.n_recv)

    def combine(self, y: torch.Tensor, stream=None, out: Optional[torch.Tensor] = None):
        """y: expert outputs, ``n_recv`` rows in receive-row order."""
        out = self.out if out is None else out
        B.ep_combine(y, self.slot, self.topk_w, self.T, self.H, self.k, out,
                     self.combine_sms, self.copy_status, stream, recv_rows=self.n_recv)
        return out

    def activation(self, gate_up: torch.Tensor, act: torch.Tensor,
                   act_scale: Optional[torch.Tensor], stream=None):
        """silu(gate) * up of the filled receive rows (the counts of the last
        layout, read on the device); ``gate_up`` bf16 [n_recv, 2I], ``act``
        e4m3 [n_recv, I] with ``act_scale`` fp32 [n_recv, I/128], or bf16
        [n_recv, I] with ``act_scale`` None."""
        I = gate_up.shape[1] // 2
        B.ep_silu_mul(gate_up, self.n_recv, I, self.expert_off, self.cnt_expert, self.P,
                      act_scale is not None, act, act_scale, self.num_sms, stream)

    def step(self, x, logits, bias, y, stream=None, out=None):
        """route, layout, dispatch (one call), then combine of the expert
        outputs y."""
        self.route_dispatch(logits, bias, x, stream)
        return self.combine(y, stream, out)

    def fused_route_dispatch(self) -> bool:
        """Whether route_dispatch runs as one kernel (mirrors the library's
        rule: T*k <= 4096, P <= 1024, at most 8 tokens per SM, the block's
        rows within one TMA transaction and 200 KB of shared memory)."""
        T, k, P, H = self.T, self.k, self.P, self.H
        if T <= 0 or T * k > 4096 or P > 1024:
            return False
        sms = torch.cuda.get_device_properties(self.recv_x.device).multi_processor_count
        if self.dispatch_sms > 0:
            sms = min(sms, self.dispatch_sms)
        tpb = -(-T // sms)
        if tpb > 8 or tpb * 2 * H >= 1 << 20:
            return False
        xb = tpb * 2 * H + (tpb * H + tpb * (H // 128) * 4 if self.fp8 else 0)
        xb = (xb + 15) // 16 * 16
        return xb + 4 * (3 * P + 1 + T * k) <= 200 * 1024

    def kernels_per_step(self) -> int:
        """Kernels one step launches: route, layout (count + slot, plus a
        column scan above 64 tiles), dispatch, combine.  Mirrors the tiling
        rule of the layout (64..512 tokens per tile, at most 64 tiles while
        tiles can grow, capped by the slot kernel's shared memory)."""
        if self.T == 0:
            return 1
        if self.fused_route_dispatch():
            return 2  # route + layout + dispatch in one kernel, combine
        if self.T * self.k <= 4096 and self.P <= 1024:
            return 3  # fused route + layout, dispatch, combine
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


class EpHostPipeline:
    """Runs batches that live in pinned host memory through an ``EpPath``
    with the PCIe copies overlapped: while batch i computes, batch i+1's
    inputs travel host -> device on one copy stream and batch i-1's result
    travels device -> host on another.  Inputs and outputs are double
    buffered on the device; the path's intermediate buffers are shared
    because the compute stream runs one batch after the other.
    """

    def __init__(self, path: EpPath, device="cuda"):
        dev = torch.device(device)
        self.path = path
        T, H, E = path.T, path.H, path.E
        self.x = [torch.empty((T, H), device=dev, dtype=torch.bfloat16) for _ in range(2)]
        self.logits = [torch.empty((T, E), device=dev, dtype=torch.float32) for _ in range(2)]
        self.bias = [torch.empty(E, device=dev, dtype=torch.float32) for _ in range(2)]
        self.out = [torch.empty((T, H), device=dev, dtype=torch.bfloat16) for _ in range(2)]
        self.s_h2d = torch.cuda.Stream(dev)
        self.s_comp = torch.cuda.Stream(dev)
        self.s_d2h = torch.cuda.Stream(dev)
        ev = lambda: [torch.cuda.Event() for _ in range(2)]  # noqa: E731
        self.h2d_done, self.comp_done, self.d2h_done = ev(), ev(), ev()

    def run(self, x_host, logits_host, bias_host, out_host, y):
        """Enqueues every batch i: x_host[i], logits_host[i], bias_host[i]
        (pinned CPU tensors) in, out_host[i] (pinned) out, with the expert
        outputs ``y`` already on the device.  Returns without synchronising;
        ``self.s_d2h`` carries the last copy."""
        p = self.path
        for i in range(len(x_host)):
            b = i & 1
            with torch.cuda.stream(self.s_h2d):
                if i >= 2:  # buffer b was read by batch i-2's compute
                    self.s_h2d.wait_event(self.comp_done[b])
                self.x[b].copy_(x_host[i], non_blocking=True)
                self.logits[b].copy_(logits_host[i], non_blocking=True)
                self.bias[b].copy_(bias_host[i], non_blocking=True)
                self.h2d_done[b].record(self.s_h2d)
            self.s_comp.wait_event(self.h2d_done[b])
            if i >= 2:      # out[b] was read by batch i-2's download
                self.s_comp.wait_event(self.d2h_done[b])
            with torch.cuda.stream(self.s_comp):
                p.step(self.x[b], self.logits[b], self.bias[b], y, stream=self.s_comp,
                       out=self.out[b])
                self.comp_done[b].record(self.s_comp)
            self.s_d2h.wait_event(self.comp_done[b])
            with torch.cuda.stream(self.s_d2h):
                out_host[i].copy_(self.out[b], non_blocking=True)
                self.d2h_done[b].record(self.s_d2h)


class EpMicroBatchPipeline:
    """Micro-batches in flight, as in the two-micro-batch overlap of
    DeepSeek's and Perplexity's EP deployments.

    Routing and layout (arithmetic- and latency-bound) run on one stream.
    With ``split_sms=None`` dispatch and combine of a batch follow each other
    on a second stream, overlapping later batches' routing.  With
    ``split_sms=(d, c)`` they get a stream each and are capped to d and c SMs,
    so the write-heavy dispatch of batch i+1 runs next to the read-heavy
    combine of batch i and HBM sees a mix of reads and writes instead of a
    pure write phase followed by a pure read phase.  Batch i uses buffer set
    i mod ``n_sets`` (one ``EpPath`` each) and starts its routing only after
    batch i - n_sets has finished its combine.  With three sets the routing
    of a batch is released together with the dispatch two batches earlier,
    every time, so the two share the GPU the same way in every step (with two
    sets the routing's start drifts against the dispatch and the step time
    moves between two levels).
    """

    def __init__(self, make_path, device="cuda", split_sms=None, n_sets: int = 3):
        if n_sets < 2:
            raise ValueError("n_sets must be at least 2")
        dev = torch.device(device)
        self.paths = [make_path() for _ in range(n_sets)]
        self.split = split_sms
        if split_sms is not None:
            for p in self.paths:
                p.dispatch_sms, p.combine_sms = split_sms
        self.s_route = torch.cuda.Stream(dev)
        self.s_move = torch.cuda.Stream(dev)     # dispatch (and combine unless split)
        self.s_comb = torch.cuda.Stream(dev) if split_sms is not None else self.s_move
        ev = lambda: [torch.cuda.Event() for _ in range(n_sets)]  # noqa: E731
        self.layout_done, self.disp_done, self.move_done = ev(), ev(), ev()

    @property
    def s_last(self):
        """the stream that carries the last combine"""
        return self.s_comb

    def run(self, xs, logits, biases, ys):
        """Enqueues batch i = (xs[i], logits[i], biases[i], expert outputs
        ys[i]); results land in ``self.paths[i % n_sets].out``.  Returns
        without synchronising; ``self.s_last`` carries the last combine."""
        n = len(self.paths)
        for i in range(len(xs)):
            b = i % n
            p = self.paths[b]
            if i >= n:  # buffer set b is free once batch i-n has combined
                self.s_route.wait_event(self.move_done[b])
            with torch.cuda.stream(self.s_route):
                p.route_layout(logits[i], biases[i], stream=self.s_route)
                self.layout_done[b].record(self.s_route)
            self.s_move.wait_event(self.layout_done[b])
            with torch.cuda.stream(self.s_move):
                p.dispatch(xs[i], stream=self.s_move)
                self.disp_done[b].record(self.s_move)
            self.s_comb.wait_event(self.disp_done[b])
            with torch.cuda.stream(self.s_comb):
                p.combine(ys[i], stream=self.s_comb)
                self.move_done[b].record(self.s_comb)

    def check_status(self):
        for p in self.paths:
            p.check_status()
