"""The one-call decode path (ep_route_dispatch) against the oracle.

Routing indices and weights, every layout array, the FP8 payload and scales
(or the BF16 rows) must be bit-identical to the oracle's route -> layout ->
dispatch on the same seeded inputs; receive rows that no slot names must be
left untouched.  The single fused kernel serves batches with T*k <= 4096;
the cases below cover it at the decode workload's own size and at ragged
and edge sizes, with replicas, the GEMM layout, an SM cap that switches to
the two-call fallback, CUDA-graph replay with new inputs, and the bounded
waits made to give up on purpose (failure detection).
"""

import numpy as np
import pytest
import torch

import oracle
from gen import CONFIGS, Workload, device_normal_bf16
from tests._common import (LAYOUT_FIELDS, gpu_layout_dict, make_path, oracle_layout,
                           oracle_route, u16)

pytestmark = pytest.mark.gpu

SENTINEL = 0xA5


@pytest.fixture(scope="module", autouse=True)
def cuda_ready():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from combine_ep_route_02_b200 import build
    build.build()
    yield
    torch.cuda.synchronize()


def fresh_path(cfg, wl, **kw):
    path = make_path(cfg, wl, **kw)
    path.recv_x.view(torch.uint8).fill_(SENTINEL)
    if path.recv_scale is not None:
        path.recv_scale.fill_(-7.0)
    for n in LAYOUT_FIELDS:
        getattr(path, n).fill_(-3 if n != "in_rank" else 9)
    path.dev_status.fill_(-1)
    return path


def check_against_oracle(cfg, wl, path, row_align=1):
    idx, w, hard = oracle_route(cfg, wl)
    assert hard.sum() == 0
    assert np.array_equal(path.topk_idx.cpu().numpy(), idx)
    assert np.array_equal(path.topk_w.cpu().numpy().view(np.uint32), w.view(np.uint32))
    lay = oracle_layout(cfg, wl, idx, row_align=row_align)
    got = gpu_layout_dict(path)
    for n in LAYOUT_FIELDS:
        g = got[n].reshape(-1)[: lay[n].size].reshape(lay[n].shape)
        assert np.array_equal(g, lay[n]), n
    assert int(path.dev_status.item()) == lay["status"] == 0
    n = path.n_recv
    rx, rs = oracle.dispatch(wl.x, lay["slot"], cfg.fp8, n_rows=n)
    named = np.zeros(n, bool)
    named[lay["slot"][lay["slot"] >= 0]] = True
    if cfg.fp8:
        gx = path.recv_x.view(torch.uint8).cpu().numpy()
        gs = path.recv_scale.cpu().numpy()
        assert np.array_equal(gx[named], rx[named])
        assert np.array_equal(gs[named].view(np.uint32), rs[named].view(np.uint32))
        assert (gx[~named] == SENTINEL).all() and (gs[~named] == -7.0).all()
    else:
        gx = u16(path.recv_x)
        assert np.array_equal(gx[named], rx[named])
        assert (gx[~named] == (SENTINEL << 8 | SENTINEL)).all()
    return idx, w, lay


def run_fused(cfg, wl, **kw):
    path = fresh_path(cfg, wl, **kw)
    path.route_dispatch(wl.logits.cuda(), wl.bias.cuda(), wl.x.cuda())
    torch.cuda.synchronize()
    return path


@pytest.mark.parametrize("T", [1, 77, 256])
def test_decode_workload(T):
    """the decode workload (T = 256, H = 7168, 256 experts in 8 groups over
    32 ranks, top-8, FP8) and ragged batch sizes below it"""
    cfg = CONFIGS["v3_decode"].scaled(T)
    wl = Workload(cfg, seed=T)
    path = run_fused(cfg, wl)
    assert path.fused_route_dispatch()
    check_against_oracle(cfg, wl, path)


@pytest.mark.parametrize("name,T", [("tiny", 128), ("tiny", 5), ("ds16b", 300), ("ds16b", 682),
                                    ("skew", 200), ("skew", 449), ("v3", 512), ("v3", 148),
                                    ("v3", 149)])
def test_other_shapes(name, T):
    """BF16 rows (tiny), k = 6 without groups (ds16b), replicas over 288
    physical experts and 32 ranks (skew), 4096 pairs with 4 tokens per block
    (v3, T = 512), and one token per SM either side of 148"""
    cfg = CONFIGS[name].scaled(T)
    wl = Workload(cfg, seed=T + 1)
    path = run_fused(cfg, wl)
    assert path.fused_route_dispatch()
    check_against_oracle(cfg, wl, path)


@pytest.mark.parametrize("R", [128, 256])
def test_many_ranks(R):
    """128 and 256 logical ranks (tokens per rank counted by a warp per rank,
    shared out over the blocks)"""
    import dataclasses
    cfg = dataclasses.replace(CONFIGS["v3_decode"].scaled(200), R=R)
    wl = Workload(cfg, seed=R)
    path = run_fused(cfg, wl)
    assert path.fused_route_dispatch()
    check_against_oracle(cfg, wl, path)


def test_largest_instance():
    """1024 experts in 32 groups, 8 kept, top-32 (the kernel instance with 32
    experts per lane), H = 512, with a 64-row tile"""
    import dataclasses
    cfg = dataclasses.replace(CONFIGS["v3_decode"].scaled(100), H=512, E=1024, R=16,
                              n_group=32, topk_group=8, topk=32)
    wl = Workload(cfg, seed=7)
    path = run_fused(cfg, wl, row_align=64)
    assert path.fused_route_dispatch()
    check_against_oracle(cfg, wl, path, row_align=64)


@pytest.mark.parametrize("A", [16, 128])
def test_gemm_layout(A):
    """each expert's rows start on a multiple of the row tile; padding rows
    get src = -1 and are not written"""
    cfg = CONFIGS["v3_decode"]
    wl = Workload(cfg, seed=A)
    path = run_fused(cfg, wl, row_align=A)
    check_against_oracle(cfg, wl, path, row_align=A)


@pytest.mark.parametrize("num_sms", [1, 20, 40, 147])
def test_sm_cap(num_sms):
    """an SM cap raises the tokens per block; above 8 tokens per block the
    call runs the two-call kernels instead, with the same results"""
    cfg = CONFIGS["v3_decode"]
    wl = Workload(cfg, seed=num_sms)
    path = run_fused(cfg, wl, num_sms=num_sms)
    assert path.fused_route_dispatch() == (num_sms >= 32)
    check_against_oracle(cfg, wl, path)


def test_larger_batch_falls_back():
    cfg = CONFIGS["v3"].scaled(600)  # 4800 pairs
    wl = Workload(cfg, seed=3)
    path = run_fused(cfg, wl)
    assert not path.fused_route_dispatch()
    check_against_oracle(cfg, wl, path)


def test_bad_replica_map_sets_status():
    """a replica count outside [1, max_rep] is reported and its pairs get
    slot -1, as in the separate layout call"""
    cfg = CONFIGS["skew"].scaled(200)
    wl = Workload(cfg, seed=8)
    idx, _, _ = oracle_route(cfg, wl)
    n_rep = wl.n_rep.clone()
    n_rep[int(idx[9, 1])] = 0
    path = fresh_path(cfg, wl)
    path.n_rep.copy_(n_rep)
    path.route_dispatch(wl.logits.cuda(), wl.bias.cuda(), wl.x.cuda())
    torch.cuda.synchronize()
    ref = oracle.layout(idx, cfg.E, cfg.n_phys, cfg.R, wl.phys_of.numpy(), n_rep.numpy())
    assert int(path.dev_status.item()) == ref["status"] == oracle.BAD_REPLICA
    got = gpu_layout_dict(path)
    for n in ("cnt_expert", "expert_off", "rows_rank", "rank_off", "tok_rank", "in_rank", "slot"):
        assert np.array_equal(got[n].reshape(ref[n].shape), ref[n]), n


def test_repeated_calls_and_graph_replay():
    """the same call repeated gives the same bytes; captured once in a CUDA
    graph with the combine and replayed over new inputs copied into the
    captured buffers, every replay matches the oracle"""
    cfg = CONFIGS["v3_decode"]
    wls = [Workload(cfg, seed=s) for s in (31, 32, 33)]
    path = fresh_path(cfg, wls[0])
    x = wls[0].x.cuda()
    lg = wls[0].logits.cuda()
    bias = wls[0].bias.cuda()
    y = device_normal_bf16(cfg.T * cfg.topk, cfg.H, seed=4)
    path.step(x, lg, bias, y)
    torch.cuda.synchronize()
    first = [t.cpu().clone() for t in (path.slot, path.recv_x.view(torch.uint8), path.out)]
    path.step(x, lg, bias, y)
    torch.cuda.synchronize()
    for a, t in zip(first, (path.slot, path.recv_x.view(torch.uint8), path.out)):
        assert torch.equal(a, t.cpu())

    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        path.step(x, lg, bias, y)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        path.step(x, lg, bias, y)
    for wl in wls[1:]:
        x.copy_(wl.x)
        lg.copy_(wl.logits)
        bias.copy_(wl.bias)
        g.replay()
        torch.cuda.synchronize()
        _, w, lay = check_against_oracle(cfg, wl, path)
        ref = oracle.combine(y.cpu(), lay["slot"], w)
        assert np.array_equal(u16(path.out), ref)
    del g


def test_waits_give_up_and_report():
    """failure detection without a fault: with the wait limit at zero every
    bounded wait (the TMA loads of the rows, the grid-wide barrier) gives up
    at once; the call returns, its status word carries EP_DEV_TIMEOUT, and
    the next call with the default limit is bit-exact"""
    from combine_ep_route_02_b200 import EP_DEV_TIMEOUT, ep_testing_set_wait_limit
    cfg = CONFIGS["v3_decode"]
    wl = Workload(cfg, seed=41)
    path = fresh_path(cfg, wl)
    x, lg, bias = wl.x.cuda(), wl.logits.cuda(), wl.bias.cuda()
    try:
        ep_testing_set_wait_limit(0)
        path.route_dispatch(lg, bias, x)
        torch.cuda.synchronize()
    finally:
        ep_testing_set_wait_limit(-1)
    assert int(path.dev_status.item()) & EP_DEV_TIMEOUT
    # the same workspace: the calls that gave up left its counters clear
    path.recv_x.view(torch.uint8).fill_(SENTINEL)
    path.recv_scale.fill_(-7.0)
    path.route_dispatch(lg, bias, x)
    torch.cuda.synchronize()
    check_against_oracle(cfg, wl, path)


def test_workspace_shared_with_the_layout_calls():
    """the route + layout calls (small-batch kernel and multi-tile kernels)
    between two fused calls on one workspace leave its counters alone"""
    cfg = CONFIGS["v3_decode"]
    wl = Workload(cfg, seed=43)
    path = fresh_path(cfg, wl)
    lg, bias, x = wl.logits.cuda(), wl.bias.cuda(), wl.x.cuda()
    path.route_dispatch(lg, bias, x)
    path.route_layout(lg, bias)
    path.layout()
    path.recv_x.view(torch.uint8).fill_(SENTINEL)
    path.recv_scale.fill_(-7.0)
    path.route_dispatch(lg, bias, x)
    torch.cuda.synchronize()
    check_against_oracle(cfg, wl, path)


def test_dispatch_tma_wait_gives_up_and_reports():
    """the TMA pipeline of ep_dispatch: with the wait limit at zero its first
    wait for a row load gives up, the CTA drains the loads in flight with the
    default limit and reports EP_DEV_TIMEOUT; the next call is bit-exact"""
    from combine_ep_route_02_b200 import EP_DEV_TIMEOUT, ep_testing_set_wait_limit
    cfg = CONFIGS["v3"].scaled(700)
    wl = Workload(cfg, seed=42)
    idx, _, _ = oracle_route(cfg, wl)
    lay = oracle_layout(cfg, wl, idx)
    path = make_path(cfg, wl)
    path.slot.copy_(torch.from_numpy(lay["slot"]))
    x = wl.x.cuda()
    path.copy_status.zero_()
    try:
        ep_testing_set_wait_limit(0)
        path.dispatch(x)
        torch.cuda.synchronize()
    finally:
        ep_testing_set_wait_limit(-1)
    assert int(path.copy_status.item()) & EP_DEV_TIMEOUT
    path.copy_status.zero_()
    path.recv_x.view(torch.uint8).fill_(0)
    path.dispatch(x)
    torch.cuda.synchronize()
    assert int(path.copy_status.item()) == 0
    rx, rs = oracle.dispatch(wl.x, lay["slot"], True)
    assert np.array_equal(path.recv_x.view(torch.uint8).cpu().numpy(), rx)
    assert np.array_equal(path.recv_scale.cpu().numpy().view(np.uint32), rs.view(np.uint32))
