"""GPU parity of the GEMM-ready path: the padded dispatch layout, dispatch and
combine over padded receive rows, and the expert activation silu(gate) * up
with its 1x128 FP8 requantisation, each against the oracle."""

import numpy as np
import pytest
import torch

import oracle
from gen import CONFIGS, Workload, device_normal_bf16

from tests._common import (LAYOUT_FIELDS, assert_combine_close, gpu_layout_dict, make_path,
                     oracle_layout, oracle_route, u16, workload)

pytestmark = pytest.mark.gpu


def assert_layout_equal(path, lay):
    got = gpu_layout_dict(path)
    n = int(lay["expert_off"][-1])
    for f in LAYOUT_FIELDS:
        g, r = got[f], lay[f]
        if f == "src":
            g = g[:n]
        assert np.array_equal(g, r), f


# ---------------------------------------------------------------------------
# padded layout
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("name,T,align", [
    ("tiny", 128, 8), ("ds16b", 4096, 64), ("v3", 8192, 128), ("skew", 16384, 128),
    ("v3", 40000, 128),           # more than 64 tiles: the column-scan kernel
    ("v3", 513, 64), ("v3_decode", 256, 128), ("skew", 300, 1024), ("ds16b", 77, 3),
])
def test_padded_layout_matches_oracle(name, T, align):
    cfg = CONFIGS[name].scaled(T)
    wl = workload(name) if T == CONFIGS[name].T else Workload(cfg, seed=T)
    idx, _, hard = oracle_route(cfg, wl)
    assert hard.sum() == 0
    lay = oracle_layout(cfg, wl, idx, row_align=align)
    a = make_path(cfg, wl, row_align=align)
    a.src.fill_(-7)
    a.route(wl.logits.cuda(), wl.bias.cuda())
    a.layout()
    torch.cuda.synchronize()
    assert np.array_equal(a.topk_idx.cpu().numpy(), idx)
    assert_layout_equal(a, lay)
    assert int(a.dev_status.item()) == 0
    # the same through ep_route_layout (one kernel for small batches)
    b = make_path(cfg, wl, row_align=align)
    b.route_layout(wl.logits.cuda(), wl.bias.cuda())
    torch.cuda.synchronize()
    assert_layout_equal(b, lay)


def test_padded_layout_empty_batch():
    cfg = CONFIGS["v3"].scaled(0)
    wl = Workload(cfg, seed=0)
    p = make_path(cfg, wl, row_align=128)
    p.expert_off.fill_(5)
    p.layout()
    torch.cuda.synchronize()
    assert int(p.expert_off.abs().sum().item()) == 0


# ---------------------------------------------------------------------------
# dispatch and combine over padded rows
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("name,T,align", [("v3", 1000, 128), ("skew", 700, 64),
                                          ("ds16b", 512, 16), ("tiny", 128, 8)])
def test_dispatch_combine_over_padded_rows(name, T, align):
    cfg = CONFIGS[name].scaled(T)
    wl = Workload(cfg, seed=11 + T)
    idx, w, _ = oracle_route(cfg, wl)
    lay = oracle_layout(cfg, wl, idx, row_align=align)
    p = make_path(cfg, wl, row_align=align)
    p.recv_x.view(torch.uint8).fill_(0xA5)
    if p.recv_scale is not None:
        p.recv_scale.fill_(-3.0)
    x = wl.x.cuda()
    p.route_layout(wl.logits.cuda(), wl.bias.cuda())
    p.dispatch(x)
    torch.cuda.synchronize()
    p.check_status()
    n = p.n_recv
    rx, rs = oracle.dispatch(wl.x, lay["slot"], cfg.fp8, n_rows=n)
    got = p.recv_x.view(torch.uint8).cpu().numpy()
    valid = np.zeros(n, bool)
    valid[lay["slot"].ravel()] = True
    ref = rx.view(np.uint8).reshape(n, -1)
    assert np.array_equal(got[valid], ref[valid])
    assert np.all(got[~valid] == 0xA5)           # padding rows are not written
    if cfg.fp8:
        gs = p.recv_scale.cpu().numpy()
        assert np.array_equal(gs[valid], rs[valid])
        assert np.all(gs[~valid] == -3.0)
    # combine reads only the pairs' rows: fill the padding with NaN
    y = device_normal_bf16(n, cfg.H, seed=5)
    y[torch.from_numpy(~valid).cuda()] = float("nan")
    out = p.combine(y)
    torch.cuda.synchronize()
    ref_out = oracle.combine(u16(y), lay["slot"], w)
    assert_combine_close(u16(out), ref_out)


# ---------------------------------------------------------------------------
# expert activation
# ---------------------------------------------------------------------------

def bits_to_bf16(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)


def same_bf16(a: np.ndarray, b: np.ndarray) -> bool:
    """bitwise equal, NaN of any payload equal to NaN"""
    na = ((a & 0x7F80) == 0x7F80) & ((a & 0x7F) != 0)
    nb = ((b & 0x7F80) == 0x7F80) & ((b & 0x7F) != 0)
    return bool(np.array_equal(na, nb) and np.array_equal(a[~na], b[~nb]))


def run_silu(gate_up_bits, fp8, expert_off=None, cnt=None, P=0, act_fill=None, sc_fill=None):
    from combine_ep_route_02_b200 import ep_silu_mul
    n, I2 = gate_up_bits.shape
    I = I2 // 2
    gu = bits_to_bf16(gate_up_bits).cuda()
    if fp8:
        act = torch.full((n, I), act_fill or 0, dtype=torch.uint8, device="cuda")
        sc = torch.full((n, I // 128), sc_fill or 0.0, dtype=torch.float32, device="cuda")
    else:
        act = torch.full((n, I), act_fill or 0, dtype=torch.int16, device="cuda")
        sc = None
    eo = None if expert_off is None else torch.from_numpy(expert_off).cuda()
    ce = None if cnt is None else torch.from_numpy(cnt).cuda()
    ep_silu_mul(gu, n, I, eo, ce, P, fp8, act, sc)
    torch.cuda.synchronize()
    a = act.cpu().numpy()
    return (a, sc.cpu().numpy()) if fp8 else (a.view(np.uint16), None)


def test_silu_every_bf16_gate_value():
    """all 65,536 gate patterns (up = 1, then up = random) in BF16 mode: h is
    bit-exact, so the SiLU rounding is checked for every input"""
    g = np.arange(65536, dtype=np.uint16).reshape(512, 128)
    silu, hard = oracle.silu_bf16_array(g)
    assert hard.sum() == 0
    one = np.full_like(g, 0x3F80)
    h, _ = run_silu(np.concatenate([g, one], axis=1), fp8=False)
    assert same_bf16(h, silu)
    rng = np.random.default_rng(3)
    up = oracle.bf16_encode_array(rng.standard_normal(g.shape).astype(np.float32) * 3)
    gu = np.concatenate([g, up], axis=1)
    h, _ = run_silu(gu, fp8=False)
    ref, _ = oracle.silu_mul_quant(gu, fp8=False)
    assert same_bf16(h, ref)
    # the same rows quantised: codes and scales bit-exact
    q, sc = run_silu(gu, fp8=True)
    q_ref, sc_ref = oracle.silu_mul_quant(gu, fp8=True)
    assert np.array_equal(q, q_ref)
    assert np.array_equal(sc.view(np.uint32), sc_ref.view(np.uint32))


@pytest.mark.parametrize("rows,I", [(1, 128), (3, 256), (37, 1408), (130, 2048), (8, 7168)])
def test_silu_mul_all_rows(rows, I):
    rng = np.random.default_rng(rows * 7 + I)
    x = rng.standard_normal((rows, 2 * I)).astype(np.float32)
    x[:, :I] *= 4.0
    gu = oracle.bf16_encode_array(x)
    q, sc = run_silu(gu, fp8=True)
    q_ref, sc_ref = oracle.silu_mul_quant(gu, fp8=True)
    assert np.array_equal(q, q_ref)
    assert np.array_equal(sc.view(np.uint32), sc_ref.view(np.uint32))


@pytest.mark.parametrize("name,T,align", [("tiny", 128, 8), ("ds16b", 700, 64),
                                          ("skew", 400, 64), ("v3", 300, 1)])
def test_silu_mul_counted_rows_only(name, T, align):
    """rows come from the layout's counts on the device; padding and tail rows
    keep their sentinel"""
    cfg = CONFIGS[name].scaled(T)
    wl = Workload(cfg, seed=T)
    idx, _, _ = oracle_route(cfg, wl)
    lay = oracle_layout(cfg, wl, idx, row_align=align)
    n = T * cfg.topk + cfg.n_phys * (align - 1)
    I = cfg.inter
    rng = np.random.default_rng(T)
    gu = oracle.bf16_encode_array(rng.standard_normal((n, 2 * I)).astype(np.float32) * 2)
    q, sc = run_silu(gu, True, lay["expert_off"], lay["cnt_expert"], cfg.n_phys, 0x5A, -9.0)
    sent_q = np.full((n, I), 0x5A, np.uint8)
    sent_s = np.full((n, I // 128), -9.0, np.float32)
    q_ref, sc_ref = oracle.silu_mul_quant(gu, True, lay["expert_off"], lay["cnt_expert"],
                                          sent_q, sent_s)
    assert np.array_equal(q, q_ref)
    assert np.array_equal(sc, sc_ref)
    assert (q[:, 0] == 0x5A).sum() >= n - T * cfg.topk


def test_silu_mul_full_size_sampled_rows():
    """V3 prefill: 8192 tokens x top-8 over a 128-row GEMM layout, I = 2048,
    through EpPath.activation; sampled rows against the oracle, every
    padding row untouched"""
    cfg = CONFIGS["v3"]
    wl = workload("v3")
    p = make_path(cfg, wl, row_align=128)
    p.route_layout(wl.logits.cuda(), wl.bias.cuda())
    I = cfg.inter
    gu = device_normal_bf16(p.n_recv, 2 * I, seed=21)
    act = torch.full((p.n_recv, I), 0x5A, dtype=torch.uint8, device="cuda")
    sc = torch.full((p.n_recv, I // 128), -9.0, dtype=torch.float32, device="cuda")
    p.activation(gu, act, sc)
    torch.cuda.synchronize()
    off = p.expert_off.cpu().numpy()
    cnt = p.cnt_expert.cpu().numpy()
    valid = np.zeros(p.n_recv, bool)
    for e in range(p.P):
        valid[off[e]:off[e] + cnt[e]] = True
    assert valid.sum() == cfg.T * cfg.topk
    a = act.cpu().numpy()
    s = sc.cpu().numpy()
    assert np.all(a[~valid] == 0x5A) and np.all(s[~valid] == -9.0)
    rows = np.random.default_rng(0).choice(np.nonzero(valid)[0], 512, replace=False)
    q_ref, s_ref = oracle.silu_mul_quant(u16(gu[torch.from_numpy(rows).cuda()]), fp8=True)
    assert np.array_equal(a[rows], q_ref)
    assert np.array_equal(s[rows], s_ref)


def test_silu_mul_graph_replay_follows_new_counts():
    """captured once, replayed after the layout changed: the launch does not
    depend on the counts, the work does"""
    cfg = CONFIGS["ds16b"].scaled(600)
    wl1, wl2 = Workload(cfg, seed=1), Workload(cfg, seed=2)
    p = make_path(cfg, wl1, row_align=64)
    I = cfg.inter
    gu = device_normal_bf16(p.n_recv, 2 * I, seed=8)
    act = torch.zeros((p.n_recv, I), dtype=torch.uint8, device="cuda")
    sc = torch.zeros((p.n_recv, I // 128), dtype=torch.float32, device="cuda")
    s = torch.cuda.Stream()
    p.route_layout(wl1.logits.cuda(), wl1.bias.cuda(), stream=s)
    p.activation(gu, act, sc, stream=s)     # first call outside capture
    s.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        p.activation(gu, act, sc, stream=s)
    for wl in (wl2, wl1):
        act.zero_()
        sc.zero_()
        p.route_layout(wl.logits.cuda(), wl.bias.cuda())
        torch.cuda.synchronize()
        g.replay()
        torch.cuda.synchronize()
        idx, _, _ = oracle_route(cfg, wl)
        lay = oracle_layout(cfg, wl, idx, row_align=64)
        q_ref, s_ref = oracle.silu_mul_quant(u16(gu), True, lay["expert_off"], lay["cnt_expert"])
        assert np.array_equal(act.cpu().numpy(), q_ref)
        assert np.array_equal(sc.cpu().numpy(), s_ref)
    del g


@pytest.mark.parametrize("T,align", [(700, 1024), (20000, 128)])
def test_padded_layout_max_sizes(T, align):
    """P = 4096, k = 32, R = 64, skewed ids, the largest row tile; T = 20000
    takes the column-scan path"""
    from combine_ep_route_02_b200 import ep_dispatch_layout, ep_workspace_size
    rng = np.random.default_rng(12)
    k, E, R = 32, 4096, 64
    idx = np.argsort(rng.random((T, E), dtype=np.float32), axis=1)[:, :k].astype(np.int32)
    idx[::3, :8] = np.arange(8)
    ref = oracle.layout(idx, E, E, R, row_align=align)
    n_src = T * k + E * (align - 1)
    d = dict(cnt_expert=E, expert_off=E + 1, rows_rank=R, rank_off=R + 1, tok_rank=R,
             slot=(T, k), src=n_src)
    g = {n: torch.full(s if isinstance(s, tuple) else (s,), -5, dtype=torch.int32,
                       device="cuda") for n, s in d.items()}
    in_rank = torch.empty((T, R), dtype=torch.uint8, device="cuda")
    ws = torch.empty(ep_workspace_size(T, k, E, R), dtype=torch.uint8, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    ep_dispatch_layout(torch.from_numpy(idx).cuda(), T, k, E, E, R, None, None, 0,
                       g["cnt_expert"], g["expert_off"], g["rows_rank"], g["rank_off"],
                       g["tok_rank"], in_rank, g["slot"], g["src"], ws, st, row_align=align)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    used = int(ref["expert_off"][-1])
    for n in d:
        got = g[n].cpu().numpy()
        if n == "src":
            assert np.all(got[used:] == -5)     # beyond the used rows: untouched
            got = got[:used]
        assert np.array_equal(got.reshape(ref[n].shape), ref[n]), n
    assert np.array_equal(in_rank.cpu().numpy(), ref["in_rank"])


def test_silu_mul_many_experts_and_gaps():
    """P = 4096 experts with synthetic counts (many empty), offsets with gaps
    between experts, and some offsets beyond the buffer: rows past the
    buffer are skipped, every other counted row matches the oracle"""
    rng = np.random.default_rng(13)
    P, I = 4096, 256
    cnt = rng.integers(0, 4, P).astype(np.int32)
    cnt[rng.random(P) < 0.5] = 0
    gaps = rng.integers(0, 3, P)
    off = np.zeros(P + 1, np.int64)
    for p in range(P):
        off[p + 1] = off[p] + cnt[p] + gaps[p]
    n_rows = int(off[P]) - 50                   # the last experts run past the buffer
    eo = off.astype(np.int32)
    gu = oracle.bf16_encode_array(rng.standard_normal((n_rows, 2 * I)).astype(np.float32))
    q, sc = run_silu(gu, True, eo, cnt, P, 0x5A, -9.0)
    sent_q = np.full((n_rows, I), 0x5A, np.uint8)
    sent_s = np.full((n_rows, I // 128), -9.0, np.float32)
    q_ref, s_ref = oracle.silu_mul_quant(gu, True, eo, cnt, sent_q, sent_s)
    assert np.array_equal(q, q_ref)
    assert np.array_equal(sc, s_ref)


def test_silu_mul_empty_counts():
    """all counts zero: nothing is written"""
    P, I, n = 64, 128, 40
    eo = np.zeros(P + 1, np.int32)
    cnt = np.zeros(P, np.int32)
    gu = np.full((n, 2 * I), 0x3F80, np.uint16)
    q, sc = run_silu(gu, True, eo, cnt, P, 0x5A, -9.0)
    assert np.all(q == 0x5A) and np.all(sc == -9.0)
