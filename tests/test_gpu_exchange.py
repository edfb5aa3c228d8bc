"""The exchange on device tensors through NCCL, in a one-rank group (the only
size a one-GPU run allows): the receive buffer goes out and comes back
unchanged, and the local combine of the returned rows matches the oracle."""

import dataclasses
import os
import socket

import numpy as np
import pytest
import torch

import oracle
from gen import CONFIGS, Workload, device_normal_bf16

from tests._common import assert_combine_close, make_path, oracle_layout, oracle_route, u16

pytestmark = pytest.mark.gpu


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_exchange_one_rank_nccl():
    import datetime

    import torch.distributed as dist

    from combine_ep_route_02_b200 import combine_exchange, dispatch_exchange, exchange_plan
    cfg = dataclasses.replace(CONFIGS["ds16b"].scaled(512), R=1)
    wl = Workload(cfg, seed=9)
    p = make_path(cfg, wl, row_align=16)
    store = dist.TCPStore("127.0.0.1", _free_port(), 1, True)
    dist.init_process_group("nccl", store=store, rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60))
    try:
        p.route_layout(wl.logits.cuda(), wl.bias.cuda())
        p.dispatch(wl.x.cuda())
        plan = exchange_plan(p.rows_rank, p.cnt_expert)
        n = int(p.rank_off[-1].item())
        assert plan.send_splits == [n] and plan.recv_splits == [n]
        assert torch.equal(plan.recv_cnt[0], p.cnt_expert.cpu().long())
        got_x = dispatch_exchange(p.recv_x, plan)
        got_s = dispatch_exchange(p.recv_scale, plan)
        torch.cuda.synchronize()
        assert torch.equal(got_x.view(torch.uint8), p.recv_x[:n].view(torch.uint8))
        assert torch.equal(got_s, p.recv_scale[:n])
        y = device_normal_bf16(n, cfg.H, seed=4)
        y_back = torch.empty((p.n_recv, cfg.H), dtype=torch.bfloat16, device="cuda")
        combine_exchange(y, plan, out=y_back)
        out = p.combine(y_back)
        torch.cuda.synchronize()
        assert torch.equal(y_back[:n], y)
        idx, w, _ = oracle_route(cfg, wl)
        lay = oracle_layout(cfg, wl, idx, row_align=16)
        assert_combine_close(u16(out), oracle.combine(u16(y_back), lay["slot"], w))
    finally:
        dist.destroy_process_group()
