"""Expert parallelism over peer memory, with every rank on this GPU.

W ranks each route and lay out their own tokens (R = W); the peer calls then
all-gather the counts, store every quantised row straight into the owning
rank's receive buffer and gather the expert outputs back.  On one GPU the
ranks' buffers are separate allocations addressed through the same
rank-indexed tables a multi-GPU group uses, and each call covers every rank
in one launch.  The receive buffers must hold, bit for bit, the oracle's
rows of every source in the documented order (expert, then source, then the
source's own order, each expert starting on a multiple of the row tile), and
each source's combine must equal the oracle's combine of the rows it gets
back.
"""

import dataclasses

import numpy as np
import pytest
import torch

import oracle
from gen import CONFIGS, Workload, device_normal_bf16
from tests._common import make_path, oracle_layout, oracle_route, u16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def cuda_ready():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from combine_ep_route_02_b200 import build
    build.build()
    yield
    torch.cuda.synchronize()


def round_up(n, a):
    return (n + a - 1) // a * a


def expected(cfgs, wls, W, A):
    """oracle layouts of every source and where each of their rows lands"""
    lays, ws = [], []
    for cfg, wl in zip(cfgs, wls):
        idx, w, _ = oracle_route(cfg, wl)
        lays.append(oracle_layout(cfg, wl, idx))
        ws.append(w)
    P = cfgs[0].n_phys
    epr = P // W
    C = np.stack([lay["cnt_expert"] for lay in lays])  # [W sources, P]
    tot = np.array([round_up(int(c), A) for c in C.sum(0)])
    start = np.zeros(P, np.int64)
    for q in range(W):
        acc = 0
        for e in range(epr):
            start[q * epr + e] = acc
            acc += tot[q * epr + e]
    dest_off = np.stack([start + C[:s].sum(0) for s in range(W)])  # [W, P]
    recv_rows = [int(tot[q * epr:(q + 1) * epr].sum()) for q in range(W)]
    return lays, ws, C, dest_off, recv_rows


def row_of(lay, dest_off_s, s_loc, epr):
    p = int(np.searchsorted(lay["expert_off"], s_loc, side="right")) - 1
    return p // epr, int(dest_off_s[p] + s_loc - lay["expert_off"][p])


def run_and_check(cfgs, wls, W, A, grp=None, seed=0):
    from combine_ep_route_02_b200 import EpPeerRanks
    paths = [make_path(c, w) for c, w in zip(cfgs, wls)]
    for p, w in zip(paths, wls):
        p.route_layout(w.logits.cuda(), w.bias.cuda())
    if grp is None:
        grp = EpPeerRanks.local(paths, cfgs[0].H, row_align=A)
    else:
        grp.paths = paths
    xs = [w.x.cuda() for w in wls]
    outs = [torch.empty((c.T, c.H), dtype=torch.bfloat16, device="cuda") for c in cfgs]
    grp.set_inputs(xs, outs)
    for t in grp.recv_x:
        t.fill_(0x5A)
    ys = [device_normal_bf16(grp.cap, cfgs[0].H, seed=seed * 10 + q) for q in range(W)]

    def experts(i, recv_x, recv_scale, y):
        y.copy_(ys[i])

    grp.step(experts)
    torch.cuda.synchronize()
    assert grp.check_status() == [0] * W

    lays, wts, C, dest_off, recv_rows = expected(cfgs, wls, W, A)
    P = cfgs[0].n_phys
    epr = P // W
    for s in range(W):
        assert np.array_equal(grp.dest_off[s].cpu().numpy(), dest_off[s])
        pd = grp.pair_dest[s].cpu().numpy()
        for (t, j), s_loc in np.ndenumerate(lays[s]["slot"]):
            assert tuple(pd[t, j]) == row_of(lays[s], dest_off[s], s_loc, epr)
        assert int(grp.recv_rows[s].item()) == recv_rows[s]
        assert np.array_equal(grp.recv_cnt[s].cpu().numpy(), C[:, s * epr:(s + 1) * epr].T)
    # every destination row holds the oracle's row of its source
    got_x = [t.cpu().numpy() for t in grp.recv_x]
    got_s = [t.cpu().numpy() for t in grp.recv_scale]
    written = [np.zeros(grp.cap, bool) for _ in range(W)]
    for s in range(W):
        rx, rs = oracle.dispatch(wls[s].x, lays[s]["slot"], True)
        for s_loc in range(int(lays[s]["expert_off"][-1])):
            q, row = row_of(lays[s], dest_off[s], s_loc, epr)
            assert np.array_equal(got_x[q][row], rx[s_loc]), (s, s_loc, q, row)
            assert np.array_equal(got_s[q][row].view(np.uint32), rs[s_loc].view(np.uint32))
            written[q][row] = True
    for q in range(W):  # padding and unused rows untouched
        assert (got_x[q][~written[q]] == 0x5A).all()
        assert written[q].sum() == C[:, q * epr:(q + 1) * epr].sum()
    # each source's combine of the rows it gets back
    ys_h = [u16(y) for y in ys]
    for s in range(W):
        n_loc = int(lays[s]["expert_off"][-1])
        y_loc = np.zeros((n_loc, cfgs[s].H), np.uint16)
        for s_loc in range(n_loc):
            q, row = row_of(lays[s], dest_off[s], s_loc, epr)
            y_loc[s_loc] = ys_h[q][row]
        ref = oracle.combine(y_loc, lays[s]["slot"], wts[s])
        assert np.array_equal(u16(outs[s]), ref), s
    return grp


def test_peer_step_other_shape():
    """the DeepSeek-16B shape (64 experts without groups, top-6, H = 2048)
    over 4 ranks with a 32-row tile, ranks of very different sizes"""
    W, A = 4, 32
    base = CONFIGS["ds16b"]
    cfgs = [dataclasses.replace(base.scaled(T), R=W) for T in (1, 300, 57, 512)]
    wls = [Workload(c, seed=90 + r) for r, c in enumerate(cfgs)]
    run_and_check(cfgs, wls, W, A, seed=4)


@pytest.mark.parametrize("W,A", [(4, 1), (4, 16), (8, 1)])
def test_peer_step_matches_oracle(W, A):
    """DeepSeek-V3 routing (256 experts, 8 groups, top-8) over W ranks, a
    different batch per rank; two steps in a row through the same buffers
    (the control words count the steps)"""
    base = CONFIGS["v3"]
    cfgs = [dataclasses.replace(base.scaled(96 + 29 * r), R=W) for r in range(W)]
    wls = [Workload(c, seed=40 + r) for r, c in enumerate(cfgs)]
    grp = run_and_check(cfgs, wls, W, A, seed=1)
    wls2 = [Workload(c, seed=60 + r) for r, c in enumerate(cfgs)]
    run_and_check(cfgs, wls2, W, A, grp=grp, seed=2)


def test_peer_waits_give_up_and_the_next_step_works():
    """with the wait limit at zero every bounded wait of the step gives up:
    each rank's status carries EP_DEV_TIMEOUT and no row is stored; with the
    default limit the next step is exact again"""
    from combine_ep_route_02_b200 import (EP_DEV_TIMEOUT, EpPeerRanks,
                                          ep_testing_set_wait_limit)
    W = 4
    base = CONFIGS["v3"]
    cfgs = [dataclasses.replace(base.scaled(64), R=W) for _ in range(W)]
    wls = [Workload(c, seed=80 + r) for r, c in enumerate(cfgs)]
    paths = [make_path(c, w) for c, w in zip(cfgs, wls)]
    for p, w in zip(paths, wls):
        p.route_layout(w.logits.cuda(), w.bias.cuda())
    grp = EpPeerRanks.local(paths, base.H)
    xs = [w.x.cuda() for w in wls]
    outs = [torch.empty((c.T, c.H), dtype=torch.bfloat16, device="cuda") for c in cfgs]
    grp.set_inputs(xs, outs)
    for t in grp.recv_x:
        t.fill_(0x5A)
    try:
        ep_testing_set_wait_limit(0)
        grp.step(lambda i, rx, rs, y: y.zero_())
        torch.cuda.synchronize()
    finally:
        ep_testing_set_wait_limit(-1)
    assert all(st & EP_DEV_TIMEOUT for st in grp.check_status())
    assert all((t == 0x5A).all() for t in grp.recv_x)
    for st in grp.status:
        st.zero_()
    run_and_check(cfgs, wls, W, 1, grp=grp, seed=3)
