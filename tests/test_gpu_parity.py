"""CUDA path (through the C ABI) vs the CPU oracle, element by element.

Routing indices and weights, every layout array, FP8 payload bytes and
scales, and BF16 dispatch rows must be bit-identical; the BF16 combine must
lie within |d| <= 1e-3 + 1e-2 |oracle| (and is expected to be identical,
because the kernel rounds in the oracle's order).  Inputs come from the
seeded generator; nothing the oracle reads comes from the CUDA path.
"""

import numpy as np
import pytest
import torch

import oracle
from gen import CONFIGS, Workload, device_normal_bf16
from tests._common import (LAYOUT_FIELDS, assert_combine_close, gpu_layout_dict, make_path,
                           oracle_layout, oracle_route, u16, workload)

pytestmark = pytest.mark.gpu

ALL = ["tiny", "ds16b", "v3", "v3_decode", "skew"]


@pytest.fixture(scope="module", autouse=True)
def cuda_ready():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from combine_ep_route_02_b200 import build
    build.build()
    yield
    torch.cuda.synchronize()


def check_route(cfg, wl, gidx, gw):
    """every token bit for bit, those whose sigmoids lie near an fp32
    rounding midpoint ("hard") included; returns how many tokens are hard"""
    idx, w, hard = oracle_route(cfg, wl)
    assert np.array_equal(gidx, idx)
    assert np.array_equal(gw.view(np.uint32), w.view(np.uint32))
    return int(hard.sum())


# ---------------------------------------------------------------------------
# routing
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("name", ALL)
def test_route_full_size(name):
    cfg = CONFIGS[name]
    wl = workload(name)
    path = make_path(cfg, wl)
    path.route(wl.logits.cuda(), wl.bias.cuda())
    torch.cuda.synchronize()
    n_hard = check_route(cfg, wl, path.topk_idx.cpu().numpy(), path.topk_w.cpu().numpy())
    assert n_hard <= 2


ROUTE_SHAPES = [  # E, G, Kg, k
    (16, 1, 1, 2), (30, 1, 1, 3), (64, 1, 1, 6), (128, 4, 2, 8), (132, 2, 1, 7),
    (256, 8, 4, 8), (288, 8, 3, 9), (512, 16, 4, 8), (1024, 32, 8, 32), (24, 3, 2, 5),
    (256, 32, 1, 8), (96, 32, 32, 32),
]


@pytest.mark.parametrize("E,G,Kg,k", ROUTE_SHAPES)
@pytest.mark.parametrize("kind", ["normal", "grid", "nobias"])
def test_route_shapes(E, G, Kg, k, kind):
    rng = np.random.default_rng(E * 7 + G * 3 + k)
    T = 203
    if kind == "grid":  # frequent exact ties among keys and group scores
        logits = rng.choice([-1.0, 0.0, 1.0], size=(T, E)).astype(np.float32)
    else:
        logits = rng.normal(0, 1, (T, E)).astype(np.float32)
    bias = None if kind == "nobias" else rng.uniform(-0.1, 0.1, E).astype(np.float32)
    for scale, renorm in [(2.5, True), (1.0, False)]:
        from combine_ep_route_02_b200 import RouteCfg, ep_route
        cfg = RouteCfg(E, G, Kg, k, scale, int(renorm))
        lg = torch.from_numpy(logits).cuda()
        bs = None if bias is None else torch.from_numpy(bias).cuda()
        gidx = torch.empty((T, k), dtype=torch.int32, device="cuda")
        gw = torch.empty((T, k), dtype=torch.float32, device="cuda")
        ep_route(lg, bs, T, cfg, gidx, gw)
        idx, w, _ = oracle.route(logits, bias, G, Kg, k, scale, renorm)
        gi, gwn = gidx.cpu().numpy(), gw.cpu().numpy()
        assert np.array_equal(gi, idx)
        assert np.array_equal(gwn.view(np.uint32), w.view(np.uint32))


def test_route_sigmoid_every_expert():
    """one group, k = E, no renorm, scale 1: the weights are the fp32
    sigmoids themselves, so every one is compared with the oracle's fp64
    evaluation (saturation, underflow and infinities included)"""
    from combine_ep_route_02_b200 import RouteCfg, ep_route
    rng = np.random.default_rng(21)
    E, T = 32, 65536
    edges = np.array([0.0, -0.0, 1e-30, -1e-30, 17.0, 17.33, -17.0, 88.0, -88.0, -87.3,
                      -103.28, -103.3, -103.97, -104.0, -110.0, 700.0, -700.0, 701.0,
                      -701.0, 1e30, -1e30, np.inf, -np.inf], np.float32)
    logits = np.concatenate([
        rng.normal(0, 1, T * E // 2), rng.normal(0, 8, T * E // 4),
        rng.uniform(-110, 110, T * E // 4 - edges.size)]).astype(np.float32)
    logits = np.concatenate([logits, edges]).reshape(T, E)
    cfg = RouteCfg(E, 1, 1, E, 1.0, 0)
    gidx = torch.empty((T, E), dtype=torch.int32, device="cuda")
    gw = torch.empty((T, E), dtype=torch.float32, device="cuda")
    ep_route(torch.from_numpy(logits).cuda(), None, T, cfg, gidx, gw)
    idx, w, _ = oracle.route(logits, None, 1, 1, E, 1.0, False)
    assert np.array_equal(gidx.cpu().numpy(), idx)
    assert np.array_equal(gw.cpu().numpy().view(np.uint32), w.view(np.uint32))


def hard_sigmoid_inputs():
    import os
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden",
                        "sigmoid_hard_inputs.txt")
    bits = [int(ln, 16) for ln in open(path) if ln.strip() and not ln.startswith("#")]
    return np.array(bits, np.uint32).view(np.float32)


def test_route_sigmoid_hard_inputs():
    """every fp32 input whose sigmoid lies within 2^-47 of an fp32 rounding
    midpoint in fp64 (the committed list): the kernel's sigmoid (one group,
    k = E, no renorm, scale 1, so the weights are the sigmoids) equals the
    oracle's correctly rounded one, bit for bit"""
    from combine_ep_route_02_b200 import RouteCfg, ep_route
    x = hard_sigmoid_inputs()
    E = 32
    n = -(-x.size // E) * E
    logits = np.resize(x, n).reshape(-1, E)
    T = logits.shape[0]
    cfg = RouteCfg(E, 1, 1, E, 1.0, 0)
    gidx = torch.empty((T, E), dtype=torch.int32, device="cuda")
    gw = torch.empty((T, E), dtype=torch.float32, device="cuda")
    ep_route(torch.from_numpy(logits).cuda(), None, T, cfg, gidx, gw)
    idx, w, hard = oracle.route(logits, None, 1, 1, E, 1.0, False)
    assert hard.all()
    assert np.array_equal(gidx.cpu().numpy(), idx)
    assert np.array_equal(gw.cpu().numpy().view(np.uint32), w.view(np.uint32))
    # the same inputs among ordinary logits through group-limited routing,
    # renormalised and scaled, on the one-kernel decode path and the
    # separate routing kernel
    from combine_ep_route_02_b200 import ep_route_dispatch  # noqa: F401
    cfg = CONFIGS["v3_decode"].scaled(96)
    wl = Workload(cfg, seed=5)
    lg = wl.logits.clone().numpy()
    flat = lg.reshape(-1)
    pos = np.random.default_rng(3).choice(flat.size, x.size, replace=False)
    flat[pos] = x
    wl.logits = torch.from_numpy(lg)
    idx, w, hard = oracle_route(cfg, wl)
    assert hard.any()
    for fused in (True, False):
        path = make_path(cfg, wl)
        if fused:
            path.route_dispatch(wl.logits.cuda(), wl.bias.cuda(), wl.x.cuda())
        else:
            path.route(wl.logits.cuda(), wl.bias.cuda())
        torch.cuda.synchronize()
        assert np.array_equal(path.topk_idx.cpu().numpy(), idx)
        assert np.array_equal(path.topk_w.cpu().numpy().view(np.uint32), w.view(np.uint32))


def test_route_empty_and_single():
    from combine_ep_route_02_b200 import RouteCfg, ep_route
    cfg = RouteCfg(256, 8, 4, 8, 2.5, 1)
    gidx = torch.full((1, 8), -7, dtype=torch.int32, device="cuda")
    gw = torch.zeros((1, 8), dtype=torch.float32, device="cuda")
    ep_route(torch.empty((0, 256), device="cuda"), None, 0, cfg, gidx, gw)
    torch.cuda.synchronize()
    assert (gidx == -7).all()
    lg = torch.randn((1, 256), generator=torch.Generator().manual_seed(3))
    ep_route(lg.cuda(), None, 1, cfg, gidx, gw)
    idx, w, _ = oracle.route(lg, None, 8, 4, 8, 2.5, True)
    assert np.array_equal(gidx.cpu().numpy(), idx)
    assert np.array_equal(gw.cpu().numpy().view(np.uint32), w.view(np.uint32))


# ---------------------------------------------------------------------------
# layout
# ---------------------------------------------------------------------------

def run_layout(cfg, wl, topk_idx_np):
    path = make_path(cfg, wl)
    path.topk_idx.copy_(torch.from_numpy(topk_idx_np))
    path.layout()
    torch.cuda.synchronize()
    return path


@pytest.mark.parametrize("name", ALL)
def test_layout_full_size(name):
    cfg = CONFIGS[name]
    wl = workload(name)
    idx, _, _ = oracle_route(cfg, wl)
    path = run_layout(cfg, wl, idx)
    ref = oracle_layout(cfg, wl, idx)
    got = gpu_layout_dict(path)
    assert ref["status"] == 0 and int(path.dev_status.item()) == 0
    for n in LAYOUT_FIELDS:
        assert np.array_equal(got[n].reshape(ref[n].shape), ref[n]), n


@pytest.mark.parametrize("T", [1, 2, 63, 64, 65, 127, 1000, 4096, 4097, 5440, 5441, 40000])
@pytest.mark.parametrize("name", ["ds16b", "skew"])
def test_layout_ragged(T, name):
    """ragged batches, and both sides of the block-size switch (tiles of at
    most 512 pairs run 512-thread blocks: top-8 up to T = 4096, top-6 up to
    T = 5440)"""
    cfg = CONFIGS[name].scaled(T)
    wl = Workload(cfg, seed=T)
    idx, _, _ = oracle_route(cfg, wl)
    path = run_layout(cfg, wl, idx)
    ref = oracle_layout(cfg, wl, idx)
    got = gpu_layout_dict(path)
    for n in LAYOUT_FIELDS:
        assert np.array_equal(got[n].reshape(ref[n].shape), ref[n]), n


def test_layout_empty():
    cfg = CONFIGS["v3"].scaled(0)
    path = make_path(cfg, Workload(cfg))
    for n in ("cnt_expert", "expert_off", "rows_rank", "rank_off", "tok_rank"):
        getattr(path, n).fill_(-5)
    path.layout()
    torch.cuda.synchronize()
    for n in ("cnt_expert", "expert_off", "rows_rank", "rank_off", "tok_rank"):
        assert (getattr(path, n) == 0).all(), n


def test_empty_batch_every_call():
    """T = 0 through every call that moves rows: each returns without
    touching its outputs, and the fused decode call writes the empty layout
    (zero counts and offsets) like ep_route_layout"""
    from combine_ep_route_02_b200 import (ep_combine, ep_combine_backward, ep_dispatch,
                                          ep_dispatch_backward)
    H, k = 7168, 8
    x = torch.empty((0, H), dtype=torch.bfloat16, device="cuda")
    slot = torch.empty((0, k), dtype=torch.int32, device="cuda")
    w = torch.empty((0, k), dtype=torch.float32, device="cuda")
    recv_x = torch.full((4, H), 0x5A, dtype=torch.uint8, device="cuda")
    recv_s = torch.full((4, H // 128), 3.0, dtype=torch.float32, device="cuda")
    y = torch.ones((4, H), dtype=torch.bfloat16, device="cuda")
    out = torch.full((1, H), 5.0, dtype=torch.bfloat16, device="cuda")
    gw = torch.full((1, k), 7.0, dtype=torch.float32, device="cuda")
    st = torch.full((1,), 9, dtype=torch.int32, device="cuda")
    ep_dispatch(x, 0, H, k, slot, True, recv_x, recv_s, dev_status=st, recv_rows=4)
    ep_combine(y, slot, w, 0, H, k, out, recv_rows=4)
    ep_dispatch_backward(y, slot, 0, H, k, out, recv_rows=4)
    ep_combine_backward(x, y, slot, w, 0, H, k, y, gw, recv_rows=4)
    torch.cuda.synchronize()
    assert (recv_x == 0x5A).all() and (recv_s == 3.0).all()
    assert (out == 5.0).all() and (y == 1.0).all() and (gw == 7.0).all()
    cfg = CONFIGS["v3_decode"].scaled(0)
    wl = Workload(cfg)
    path = make_path(cfg, wl)
    for n in ("cnt_expert", "expert_off", "rows_rank", "rank_off", "tok_rank"):
        getattr(path, n).fill_(-5)
    path.route_dispatch(wl.logits.cuda(), wl.bias.cuda(), wl.x.cuda())
    torch.cuda.synchronize()
    path.check_status()
    for n in ("cnt_expert", "expert_off", "rows_rank", "rank_off", "tok_rank"):
        assert (getattr(path, n) == 0).all(), n


@pytest.mark.parametrize("T", [700, 20000])
def test_layout_max_sizes_and_skewed_ids(T):
    """P = 4096 physical experts, k = 32, R = 64, heavily skewed expert ids;
    T = 20000 takes more tiles than the slot kernel sums itself, with the
    largest tiles its shared memory allows"""
    from combine_ep_route_02_b200 import ep_dispatch_layout, ep_workspace_size
    rng = np.random.default_rng(11)
    k, E, R = 32, 4096, 64
    idx = np.argsort(rng.random((T, E), dtype=np.float32), axis=1)[:, :k].astype(np.int32)
    idx[::3, :8] = np.arange(8)  # many tokens on the same few experts
    ref = oracle.layout(idx, E, E, R)
    d = dict(cnt_expert=E, expert_off=E + 1, rows_rank=R, rank_off=R + 1, tok_rank=R,
             slot=(T, k), src=T * k)
    g = {n: torch.empty(s, dtype=torch.int32, device="cuda") for n, s in d.items()}
    in_rank = torch.empty((T, R), dtype=torch.uint8, device="cuda")
    ws = torch.empty(ep_workspace_size(T, k, E, R), dtype=torch.uint8, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    ep_dispatch_layout(torch.from_numpy(idx).cuda(), T, k, E, E, R, None, None, 0,
                       g["cnt_expert"], g["expert_off"], g["rows_rank"], g["rank_off"],
                       g["tok_rank"], in_rank, g["slot"], g["src"], ws, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    for n in d:
        assert np.array_equal(g[n].cpu().numpy().reshape(ref[n].shape), ref[n]), n
    assert np.array_equal(in_rank.cpu().numpy(), ref["in_rank"])


def test_layout_bad_ids_set_status():
    cfg = CONFIGS["skew"].scaled(300)
    wl = Workload(cfg)
    idx, _, _ = oracle_route(cfg, wl)
    idx[5, 2] = 256        # out of range
    idx[77, 0] = -3
    path = run_layout(cfg, wl, idx)
    ref = oracle_layout(cfg, wl, idx)
    assert ref["status"] == oracle.BAD_EXPERT
    assert int(path.dev_status.item()) == ref["status"]
    got = gpu_layout_dict(path)
    for n in ("cnt_expert", "expert_off", "rows_rank", "rank_off", "tok_rank", "in_rank", "slot"):
        assert np.array_equal(got[n].reshape(ref[n].shape), ref[n]), n
    # a broken replica map is reported too, and never read out of bounds
    n_rep = wl.n_rep.clone()
    n_rep[int(idx[9, 1])] = 0
    path2 = make_path(cfg, wl)
    path2.n_rep.copy_(n_rep)
    path2.topk_idx.copy_(torch.from_numpy(idx))
    path2.layout()
    ref2 = oracle.layout(idx, cfg.E, cfg.n_phys, cfg.R, wl.phys_of.numpy(), n_rep.numpy())
    assert int(path2.dev_status.item()) == ref2["status"] == oracle.BAD_EXPERT | oracle.BAD_REPLICA
    assert np.array_equal(path2.slot.cpu().numpy(), ref2["slot"])


# ---------------------------------------------------------------------------
# dispatch
# ---------------------------------------------------------------------------

def check_dispatch(cfg, x_cpu, slot_np, path):
    rx, rs = oracle.dispatch(x_cpu, slot_np, cfg.fp8)
    if cfg.fp8:
        got = path.recv_x.view(torch.uint8).cpu().numpy()
        bad = np.nonzero((got != rx).any(axis=1))[0]
        assert bad.size == 0, (bad[:5], got[bad[0]][:16], rx[bad[0]][:16])
        gs = path.recv_scale.cpu().numpy()
        assert np.array_equal(gs.view(np.uint32), rs.view(np.uint32))
    else:
        assert np.array_equal(u16(path.recv_x), rx)


@pytest.mark.parametrize("name", ALL)
def test_dispatch_full_size(name):
    cfg = CONFIGS[name]
    wl = workload(name)
    idx, _, _ = oracle_route(cfg, wl)
    lay = oracle_layout(cfg, wl, idx)
    path = make_path(cfg, wl)
    path.slot.copy_(torch.from_numpy(lay["slot"]))
    path.dispatch(wl.x.cuda())
    torch.cuda.synchronize()
    check_dispatch(cfg, wl.x, lay["slot"], path)


def adversarial_rows(H=1024):
    """blocks that stress the quantiser: zeros, -0, tiny and huge amax,
    saturation, exact e4m3 ties after scaling, bf16 subnormals"""
    rng = np.random.default_rng(12)
    rows = []
    nb = H // 128

    def row(blocks):
        return np.concatenate(blocks).astype(np.float32)

    z = np.zeros(128, np.float32)
    rows.append(row([z] * nb))
    rows.append(row([-z] * nb))
    rows.append(row([np.full(128, 3.0, np.float32)] * nb))                     # all == amax
    ties = np.array([448.0] + [1.0625, 1.1875, -2.125, 0.0029296875, 0.0009765625] * 25 +
                    [0.5, 0.25], np.float32)                                  # scale 1: RNE ties
    rows.append(row([ties] * nb))
    rows.append(row([rng.normal(0, 1e-38, 128).astype(np.float32)] * nb))      # subnormal amax
    rows.append(row([rng.normal(0, 1e37, 128).astype(np.float32)] * nb))       # huge values
    rows.append(row([np.where(np.arange(128) == 5, 1e-30, 1e-41).astype(np.float32)] * nb))
    mix = []
    for b in range(nb):
        v = rng.normal(0, 10.0 ** rng.integers(-20, 20), 128).astype(np.float32)
        v[rng.integers(0, 128)] = 0.0
        mix.append(v)
    rows.append(row(mix))
    x = torch.from_numpy(np.stack(rows)).to(torch.bfloat16)
    # every bf16 bit pattern that is finite, in blocks with a common amax
    pats = np.arange(65536, dtype=np.uint32)
    fin = pats[((pats >> 7) & 0xFF) != 0xFF].astype(np.uint16)
    allb = torch.from_numpy(fin.view(np.int16)).view(torch.bfloat16)
    n = (allb.numel() // H) * H
    x = torch.cat([x, allb[:n].view(-1, H)])
    return x


def test_dispatch_adversarial_blocks():
    x = adversarial_rows()
    T, H, k = x.shape[0], x.shape[1], 3
    cfg = CONFIGS["v3"].scaled(T)
    rng = np.random.default_rng(13)
    slot = rng.permutation(T * k).astype(np.int32).reshape(T, k)
    from combine_ep_route_02_b200 import ep_dispatch
    rx = torch.empty((T * k, H), dtype=torch.uint8, device="cuda")
    rs = torch.empty((T * k, H // 128), dtype=torch.float32, device="cuda")
    ep_dispatch(x.cuda(), T, H, k, torch.from_numpy(slot).cuda(), True, rx, rs)
    torch.cuda.synchronize()
    ref_x, ref_s = oracle.dispatch(x, slot, True)
    assert np.array_equal(rx.cpu().numpy(), ref_x)
    assert np.array_equal(rs.cpu().numpy().view(np.uint32), ref_s.view(np.uint32))
    assert cfg.T == T


@pytest.mark.parametrize("num_sms", [1, 3, 37, 0])
def test_dispatch_num_sms_and_invalid_slots(num_sms):
    cfg = CONFIGS["ds16b"].scaled(517)
    wl = Workload(cfg, seed=5)
    idx, _, _ = oracle_route(cfg, wl)
    lay = oracle_layout(cfg, wl, idx)
    slot = lay["slot"].copy()
    slot[3, 1] = -1                 # skipped
    slot[10, 0] = cfg.T * cfg.topk  # out of range: skipped
    path = make_path(cfg, wl, num_sms=num_sms)
    path.recv_x.view(torch.uint8).fill_(0xAB)
    path.recv_scale.fill_(-1.0)
    path.slot.copy_(torch.from_numpy(slot))
    path.dispatch(wl.x.cuda())
    torch.cuda.synchronize()
    rx, rs = oracle.dispatch(wl.x, slot, True)
    got = path.recv_x.view(torch.uint8).cpu().numpy()
    gs = path.recv_scale.cpu().numpy()
    unwritten = np.setdiff1d(np.arange(cfg.T * cfg.topk), slot[slot >= 0][slot[slot >= 0] < cfg.T * cfg.topk])
    written = np.setdiff1d(np.arange(cfg.T * cfg.topk), unwritten)
    assert np.array_equal(got[written], rx[written])
    assert np.array_equal(gs[written], rs[written])
    assert (got[unwritten] == 0xAB).all() and (gs[unwritten] == -1.0).all()


@pytest.mark.parametrize("k", [1, 13, 14, 32])
def test_dispatch_tma_topk(k):
    """the TMA pipeline at H = 7168 (14 warps: warp 0 issues the code rows'
    bulk copies, the other 13 write the k scale rows, several each from
    k = 14) with invalid slots, against the oracle"""
    from combine_ep_route_02_b200 import ep_dispatch
    T, H = 97, 7168
    g = torch.Generator().manual_seed(k)
    x = (torch.randn((T, H), generator=g) * 3).to(torch.bfloat16)
    rng = np.random.default_rng(k)
    slot = rng.permutation(T * k).astype(np.int32).reshape(T, k)
    slot[0, k - 1] = -1
    slot[T - 1, 0] = T * k
    rx = torch.full((T * k, H), 0x5A, dtype=torch.uint8, device="cuda")
    rs = torch.full((T * k, H // 128), -2.0, dtype=torch.float32, device="cuda")
    ep_dispatch(x.cuda(), T, H, k, torch.from_numpy(slot).cuda(), True, rx, rs)
    torch.cuda.synchronize()
    ref_x, ref_s = oracle.dispatch(x, slot, True)
    ok = slot[(slot >= 0) & (slot < T * k)]
    untouched = np.setdiff1d(np.arange(T * k), ok)
    got_x, got_s = rx.cpu().numpy(), rs.cpu().numpy()
    assert np.array_equal(got_x[ok], ref_x[ok])
    assert np.array_equal(got_s[ok].view(np.uint32), ref_s[ok].view(np.uint32))
    assert (got_x[untouched] == 0x5A).all() and (got_s[untouched] == -2.0).all()


def test_dispatch_fp8_thread_store_path():
    """a recv_scale that is 4- but not 16-byte aligned takes the thread-store
    kernel instead of the TMA pipeline; both must give the oracle's bytes"""
    cfg = CONFIGS["v3"].scaled(300)
    wl = Workload(cfg, seed=6)
    idx, _, _ = oracle_route(cfg, wl)
    lay = oracle_layout(cfg, wl, idx)
    from combine_ep_route_02_b200 import ep_dispatch
    T, H, k = cfg.T, cfg.H, cfg.topk
    rx = torch.empty((T * k, H), dtype=torch.uint8, device="cuda")
    rs_buf = torch.empty(T * k * (H // 128) + 1, dtype=torch.float32, device="cuda")
    rs = rs_buf[1:].view(T * k, H // 128)
    assert rs.data_ptr() % 16 == 4
    ep_dispatch(wl.x.cuda(), T, H, k, torch.from_numpy(lay["slot"]).cuda(), True, rx, rs)
    torch.cuda.synchronize()
    ref_x, ref_s = oracle.dispatch(wl.x, lay["slot"], True)
    assert np.array_equal(rx.cpu().numpy(), ref_x)
    assert np.array_equal(rs.cpu().numpy().view(np.uint32), ref_s.view(np.uint32))


def test_dispatch_bf16_ragged():
    cfg = CONFIGS["tiny"].scaled(333)
    wl = Workload(cfg, seed=9)
    idx, _, _ = oracle_route(cfg, wl)
    lay = oracle_layout(cfg, wl, idx)
    path = make_path(cfg, wl, num_sms=5)
    path.slot.copy_(torch.from_numpy(lay["slot"]))
    path.dispatch(wl.x.cuda())
    torch.cuda.synchronize()
    check_dispatch(cfg, wl.x, lay["slot"], path)


# ---------------------------------------------------------------------------
# combine
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("name", ALL)
def test_combine_full_size(name):
    cfg = CONFIGS[name]
    wl = workload(name)
    idx, w, _ = oracle_route(cfg, wl)
    lay = oracle_layout(cfg, wl, idx)
    y = device_normal_bf16(cfg.T * cfg.topk, cfg.H, seed=1)
    path = make_path(cfg, wl)
    path.slot.copy_(torch.from_numpy(lay["slot"]))
    path.topk_w.copy_(torch.from_numpy(w))
    path.combine(y)
    torch.cuda.synchronize()
    ref = oracle.combine(y.cpu(), lay["slot"], w)
    got = u16(path.out)
    assert_combine_close(got, ref)
    # same rounding sequence as the oracle: expected bit-identical
    assert np.array_equal(got, ref)


@pytest.mark.parametrize("k", [1, 3, 8, 9, 17, 32])
def test_combine_topk_and_invalid_slots(k):
    rng = np.random.default_rng(20 + k)
    T, H = 257, 520
    y = device_normal_bf16(T * k, H, seed=k)
    slot = rng.permutation(T * k).astype(np.int32).reshape(T, k)
    slot[0, 0] = -1
    slot[7, k - 1] = T * k
    w = rng.uniform(-1, 2, (T, k)).astype(np.float32)
    out = torch.empty((T, H), dtype=torch.bfloat16, device="cuda")
    from combine_ep_route_02_b200 import ep_combine
    ep_combine(y, torch.from_numpy(slot).cuda(), torch.from_numpy(w).cuda(), T, H, k, out,
               num_sms=7)
    torch.cuda.synchronize()
    ref = oracle.combine(y.cpu(), slot, w)
    assert_combine_close(u16(out), ref)
    assert np.array_equal(u16(out), ref)


# ---------------------------------------------------------------------------
# whole path
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("name", ["v3", "skew", "v3_decode"])
def test_full_path(name):
    """route -> layout -> dispatch -> combine in one stream, as the bench runs it"""
    cfg = CONFIGS[name]
    wl = workload(name)
    path = make_path(cfg, wl)
    y = device_normal_bf16(cfg.T * cfg.topk, cfg.H, seed=2)
    path.step(wl.x.cuda(), wl.logits.cuda(), wl.bias.cuda(), y)
    torch.cuda.synchronize()
    idx, w, hard = oracle_route(cfg, wl)
    assert hard.sum() == 0
    assert np.array_equal(path.topk_idx.cpu().numpy(), idx)
    assert np.array_equal(path.topk_w.cpu().numpy().view(np.uint32), w.view(np.uint32))
    lay = oracle_layout(cfg, wl, idx)
    got = gpu_layout_dict(path)
    for n in LAYOUT_FIELDS:
        assert np.array_equal(got[n].reshape(lay[n].shape), lay[n]), n
    check_dispatch(cfg, wl.x, lay["slot"], path)
    ref = oracle.combine(y.cpu(), lay["slot"], w)
    assert_combine_close(u16(path.out), ref)


def test_identity_expert_round_trip():
    """dispatch -> dequantised identity experts -> combine recovers x"""
    cfg = CONFIGS["ds16b"]
    wl = Workload(cfg)
    path = make_path(cfg, wl)
    x = wl.x.cuda()
    path.route(wl.logits.cuda(), wl.bias.cuda())
    path.layout()
    path.dispatch(x)
    deq = path.recv_x.float() * path.recv_scale.repeat_interleave(128, dim=1)
    path.combine(deq.to(torch.bfloat16))
    torch.cuda.synchronize()
    xf = x.double()
    sc = xf.abs().view(cfg.T, -1, 128).amax(2).repeat_interleave(128, dim=1) / 448
    bound = (2.0 ** -4 + 2.0 ** -7) * xf.abs() + 2.0 ** -9 * sc + 1e-30
    assert ((path.out.double() - xf).abs() <= bound).all()


def test_deterministic_across_runs_and_grids():
    cfg = CONFIGS["skew"].scaled(3000)
    wl = Workload(cfg, seed=4)
    y = device_normal_bf16(cfg.T * cfg.topk, cfg.H, seed=3)
    outs = []
    for num_sms in (0, 11):
        path = make_path(cfg, wl, num_sms=num_sms)
        path.step(wl.x.cuda(), wl.logits.cuda(), wl.bias.cuda(), y)
        torch.cuda.synchronize()
        outs.append([t.cpu().clone() for t in (path.topk_idx, path.slot, path.src,
                                                path.recv_x.view(torch.uint8), path.recv_scale,
                                                path.out)])
    for a, b in zip(*outs):
        assert torch.equal(a, b)


def test_host_pipeline_overlapped_batches():
    """three different batches from pinned host memory through the
    overlapped pipeline; every result equals the oracle's"""
    from combine_ep_route_02_b200 import EpHostPipeline
    cfg = CONFIGS["v3"].scaled(300)
    wls = [Workload(cfg, seed=s) for s in (11, 12, 13)]
    path = make_path(cfg, wls[0])
    pipe = EpHostPipeline(path)
    y = device_normal_bf16(cfg.T * cfg.topk, cfg.H, seed=5)
    xs = [w.x.pin_memory() for w in wls]
    lgs = [w.logits.pin_memory() for w in wls]
    bs = [w.bias.pin_memory() for w in wls]
    outs = [torch.empty((cfg.T, cfg.H), dtype=torch.bfloat16).pin_memory() for _ in wls]
    pipe.run(xs, lgs, bs, outs, y)
    torch.cuda.synchronize()
    yc = y.cpu()
    for w, o in zip(wls, outs):
        idx, wt, hard = oracle_route(cfg, w)
        assert hard.sum() == 0
        lay = oracle_layout(cfg, w, idx)
        ref = oracle.combine(yc, lay["slot"], wt)
        assert np.array_equal(u16(o), ref)


@pytest.mark.parametrize("n_sets", [2, 3])
def test_micro_batch_pipeline(n_sets):
    """four different batches through the two-stream micro-batch schedule
    with n_sets buffer sets; every batch's layout and result equal the
    oracle's"""
    from combine_ep_route_02_b200 import EpMicroBatchPipeline
    cfg = CONFIGS["skew"].scaled(700)
    wls = [Workload(cfg, seed=s) for s in (21, 22, 23, 24)]
    pipe = EpMicroBatchPipeline(lambda: make_path(cfg, wls[0]), n_sets=n_sets)
    ys = [device_normal_bf16(cfg.T * cfg.topk, cfg.H, seed=30 + i) for i in range(4)]
    outs = []
    for i in range(4):  # one batch at a time so every result can be kept
        pipe.run([wls[i].x.cuda()], [wls[i].logits.cuda()], [wls[i].bias.cuda()], [ys[i]])
        torch.cuda.synchronize()
        p = pipe.paths[0]
        outs.append((u16(p.out), p.slot.cpu().numpy().copy()))
    # every batch is laid out with the pipeline's replica map (batch 0's)
    po, nr = wls[0].phys_of.numpy(), wls[0].n_rep.numpy()
    for w, y, (o, sl) in zip(wls, ys, outs):
        idx, wt, hard = oracle_route(cfg, w)
        assert hard.sum() == 0
        lay = oracle.layout(idx, cfg.E, cfg.n_phys, cfg.R, po, nr)
        assert np.array_equal(sl, lay["slot"])
        assert np.array_equal(o, oracle.combine(y.cpu(), lay["slot"], wt))
    # all four enqueued at once: the overlapped schedule gives the same bytes
    pipe.run([w.x.cuda() for w in wls], [w.logits.cuda() for w in wls],
             [w.bias.cuda() for w in wls], ys)
    torch.cuda.synchronize()
    pipe.check_status()
    for i in range(4 - n_sets, 4):  # the last batch of each buffer set
        assert np.array_equal(u16(pipe.paths[i % n_sets].out), outs[i][0])


@pytest.mark.parametrize("name,T", [("v3_decode", 256), ("v3_decode", 1), ("v3_decode", 77),
                                    ("tiny", 128), ("skew", 512), ("ds16b", 682),
                                    ("v3", 513), ("skew", 3000)])
def test_route_layout_fused_equals_two_calls(name, T):
    """ep_route_layout (one kernel while T*k <= 4096) gives the bytes of
    ep_route + ep_dispatch_layout and of the oracle"""
    cfg = CONFIGS[name].scaled(T)
    wl = Workload(cfg, seed=40 + T)
    a, b = make_path(cfg, wl), make_path(cfg, wl)
    lg, bs = wl.logits.cuda(), wl.bias.cuda()
    a.route(lg, bs)
    a.layout()
    b.dev_status.fill_(-1)
    b.route_layout(lg, bs)
    torch.cuda.synchronize()
    for n in ("topk_idx", "topk_w", "cnt_expert", "expert_off", "rows_rank", "rank_off",
              "tok_rank", "in_rank", "slot", "src", "dev_status"):
        assert torch.equal(getattr(a, n), getattr(b, n)), n
    idx, w, hard = oracle_route(cfg, wl)
    assert hard.sum() == 0
    assert np.array_equal(b.topk_idx.cpu().numpy(), idx)
    lay = oracle_layout(cfg, wl, idx)
    assert np.array_equal(b.slot.cpu().numpy(), lay["slot"])
    # a second call on the same workspace (the completion counter is reset)
    b.route_layout(lg, bs)
    torch.cuda.synchronize()
    assert torch.equal(a.slot, b.slot)


# ---------------------------------------------------------------------------
# backward (training)
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("name", ["v3", "ds16b", "tiny"])
def test_dispatch_backward(name):
    from combine_ep_route_02_b200 import ep_dispatch_backward
    cfg = CONFIGS[name]
    wl = workload(name)
    idx, _, _ = oracle_route(cfg, wl)
    slot = oracle_layout(cfg, wl, idx)["slot"].copy()
    slot[1, 0] = -1
    g = device_normal_bf16(cfg.T * cfg.topk, cfg.H, seed=7)
    gx = torch.empty((cfg.T, cfg.H), dtype=torch.bfloat16, device="cuda")
    ep_dispatch_backward(g, torch.from_numpy(slot).cuda(), cfg.T, cfg.H, cfg.topk, gx)
    torch.cuda.synchronize()
    ref = oracle.dispatch_backward(g.cpu(), slot)
    assert_combine_close(u16(gx), ref)
    assert np.array_equal(u16(gx), ref)


@pytest.mark.parametrize("name", ["v3", "ds16b", "skew"])
def test_combine_backward(name):
    from combine_ep_route_02_b200 import ep_combine_backward
    cfg = CONFIGS[name] if name != "skew" else CONFIGS[name].scaled(2000)
    wl = workload(name) if name != "skew" else Workload(cfg, seed=3)
    idx, w, _ = oracle_route(cfg, wl)
    slot = oracle_layout(cfg, wl, idx)["slot"].copy()
    slot[2, 3] = -1
    n = cfg.T * cfg.topk
    y = device_normal_bf16(n, cfg.H, seed=8)
    g = device_normal_bf16(cfg.T, cfg.H, seed=9)
    gy = torch.zeros((n, cfg.H), dtype=torch.bfloat16, device="cuda")
    gw = torch.empty((cfg.T, cfg.topk), dtype=torch.float32, device="cuda")
    ep_combine_backward(g, y, torch.from_numpy(slot).cuda(), torch.from_numpy(w).cuda(), cfg.T,
                        cfg.H, cfg.topk, gy, gw)
    torch.cuda.synchronize()
    ref_y, ref_w = oracle.combine_backward(g.cpu(), y.cpu(), slot, w)
    assert np.array_equal(u16(gy), ref_y)
    # fp32 dot products in a different order than the oracle's fp64 sum
    yc, gc = y.cpu().double().numpy(), g.cpu().double().numpy()
    valid = slot >= 0
    mag = np.zeros_like(ref_w, dtype=np.float64)
    mag[valid] = np.einsum("th,th->t", np.abs(gc)[np.nonzero(valid)[0]],
                           np.abs(yc[slot[valid]]))
    err = np.abs(gw.cpu().numpy().astype(np.float64) - ref_w)
    assert (err <= 1e-5 * mag + 1e-6).all(), float((err - 1e-5 * mag).max())
    assert (gw.cpu().numpy()[~valid] == 0).all()


@pytest.mark.parametrize("T,R", [(300, 128), (5000, 256)])
def test_layout_many_ranks(T, R):
    """more than 64 logical ranks: in_rank and the rank counts come from the
    per-(token, rank) path of the count phase"""
    from combine_ep_route_02_b200 import ep_dispatch_layout, ep_workspace_size
    rng = np.random.default_rng(14)
    k, E = 8, 512
    idx = np.argsort(rng.random((T, E), dtype=np.float32), axis=1)[:, :k].astype(np.int32)
    ref = oracle.layout(idx, E, E, R)
    d = dict(cnt_expert=E, expert_off=E + 1, rows_rank=R, rank_off=R + 1, tok_rank=R,
             slot=(T, k), src=T * k)
    g = {n: torch.empty(s, dtype=torch.int32, device="cuda") for n, s in d.items()}
    in_rank = torch.empty((T, R), dtype=torch.uint8, device="cuda")
    ws = torch.empty(ep_workspace_size(T, k, E, R), dtype=torch.uint8, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    ep_dispatch_layout(torch.from_numpy(idx).cuda(), T, k, E, E, R, None, None, 0,
                       g["cnt_expert"], g["expert_off"], g["rows_rank"], g["rank_off"],
                       g["tok_rank"], in_rank, g["slot"], g["src"], ws, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    for n in d:
        assert np.array_equal(g[n].cpu().numpy().reshape(ref[n].shape), ref[n]), n
    assert np.array_equal(in_rank.cpu().numpy(), ref["in_rank"])


@pytest.mark.parametrize("k,H", [(12, 2048), (32, 1024), (3, 7168)])
def test_combine_backward_topk_and_widths(k, H):
    """top-k above 8 (the general instance of the kernel) and row widths that
    give different block sizes"""
    from combine_ep_route_02_b200 import ep_combine_backward
    rng = np.random.default_rng(k * 100 + H)
    T = 97
    n = T * k
    slot = rng.permutation(n).astype(np.int32).reshape(T, k)
    slot[5, k - 1] = -1
    w = rng.uniform(0.05, 1.5, (T, k)).astype(np.float32)
    y = device_normal_bf16(n, H, seed=k)
    g = device_normal_bf16(T, H, seed=k + 1)
    gy = torch.zeros((n, H), dtype=torch.bfloat16, device="cuda")
    gw = torch.empty((T, k), dtype=torch.float32, device="cuda")
    ep_combine_backward(g, y, torch.from_numpy(slot).cuda(), torch.from_numpy(w).cuda(), T, H, k,
                        gy, gw)
    torch.cuda.synchronize()
    ref_y, ref_w = oracle.combine_backward(g.cpu(), y.cpu(), slot, w)
    assert np.array_equal(u16(gy), ref_y)
    yc, gc = y.cpu().double().numpy(), g.cpu().double().numpy()
    valid = slot >= 0
    mag = np.zeros_like(ref_w, dtype=np.float64)
    mag[valid] = np.einsum("th,th->t", np.abs(gc)[np.nonzero(valid)[0]],
                           np.abs(yc[slot[valid]]))
    err = np.abs(gw.cpu().numpy().astype(np.float64) - ref_w)
    assert (err <= 1e-5 * mag + 1e-6).all()
    assert (gw.cpu().numpy()[~valid] == 0).all()
