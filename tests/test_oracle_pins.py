"""Pins for the CPU oracle, each against something other than the oracle.

Routing: brute force over all group and expert subsets on tiny inputs, tie
suites, a worked example, torch.topk for the single-group case, invariants.
Layout: a sort-based restatement, permutation / inverse / ordering
invariants, and the counting facts the Perplexity blog prints.
FP8 / BF16 formats: torch's converters, a nearest-value search over the
decoded code table, closed-form special values.
Dispatch / combine: the per-block scale identity, the e4m3 half-ulp error
bound, an identity-expert round trip, and an fp64 restatement of the sum.
"""

import itertools
import json
import math
import os

import numpy as np
import pytest
import torch
from hypothesis import given, settings
from hypothesis import strategies as st

import oracle
from gen import CONFIGS, Workload

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")

F32 = np.float32


# ---------------------------------------------------------------------------
# independent restatements used only as pins
# ---------------------------------------------------------------------------

def sig_f32(x):
    """fp32 rounding of the fp64 logistic function, via Python's math."""
    return F32(1.0 / (1.0 + math.exp(-float(x))))


def beats(a, b):
    """total order on (value, index): larger value first, lower index on ties"""
    return a[0] > b[0] or (a[0] == b[0] and a[1] < b[1])


def top_set_bruteforce(items, n):
    """The unique n-subset whose every member beats every non-member."""
    found = []
    for comb in itertools.combinations(range(len(items)), n):
        inside = set(comb)
        if all(beats(items[i], items[o]) for i in inside for o in range(len(items))
               if o not in inside):
            found.append(comb)
    assert len(found) == 1
    return sorted(found[0], key=lambda i: (-items[i][0], items[i][1]))


def route_bruteforce(logits, bias, G, Kg, k, scale, renorm):
    E = len(logits)
    s = [sig_f32(v) for v in logits]
    key = [F32(s[e] + F32(bias[e])) for e in range(E)]
    gs = E // G
    if G > 1:
        gscore = []
        for g in range(G):
            top2 = sorted((key[e] for e in range(g * gs, (g + 1) * gs)), reverse=True)[:2]
            gscore.append((F32(top2[0] + top2[1]), g))
        groups = top_set_bruteforce(gscore, Kg)
        allowed = [e for e in range(E) if e // gs in groups]
    else:
        allowed = list(range(E))
    items = [(key[e], e) for e in allowed]
    pick = [allowed[i] for i in top_set_bruteforce(items, k)]
    w = [s[e] for e in pick]
    if renorm:
        tot = F32(0.0)
        for v in w:
            tot = F32(tot + v)
        if tot != 0:
            w = [F32(v / tot) for v in w]
    w = [F32(v * F32(scale)) for v in w]
    return pick, w


# ---------------------------------------------------------------------------
# number formats
# ---------------------------------------------------------------------------

def e4m3_table():
    """value of every finite e4m3fn code, from the format definition"""
    vals = {}
    for c in range(256):
        s, E, m = c >> 7, (c >> 3) & 15, c & 7
        if E == 15 and m == 7:
            continue
        v = m * 2.0 ** -9 if E == 0 else (1 + m / 8) * 2.0 ** (E - 7)
        vals[c] = -v if s else v
    return vals


def test_e4m3_special_values():
    enc = oracle.e4m3_encode
    assert enc(448.0) == 0x7E and enc(-448.0) == 0xFE
    assert enc(1.0) == 0x38 and enc(2.0 ** -9) == 0x01 and enc(2.0 ** -6) == 0x08
    assert enc(0.0) == 0x00 and enc(-0.0) == 0x80
    assert enc(1e30) == 0x7E and enc(float("inf")) == 0x7E and enc(-1e30) == 0xFE
    assert enc(float("nan")) == 0x7F
    # ties to even: 1 + 1/16 lies halfway between 1 (m=0) and 1.125 (m=1)
    assert enc(1.0625) == 0x38 and enc(1.1875) == 0x3A
    # halfway between 0 and the smallest subnormal rounds to 0 (even)
    assert enc(2.0 ** -10) == 0x00 and enc(3 * 2.0 ** -10) == 0x02
    # 464 is halfway between 448 and the (NaN) 480 pattern: saturates
    assert enc(464.0) == 0x7E and enc(447.9) == 0x7E


def test_e4m3_decode_roundtrip():
    tab = e4m3_table()
    assert len(tab) == 254
    for c, v in tab.items():
        assert oracle.e4m3_decode(c) == pytest.approx(v, abs=0)
        assert oracle.e4m3_encode(v) == c
    assert math.isnan(oracle.e4m3_decode(0x7F)) and math.isnan(oracle.e4m3_decode(0xFF))


def _structured_f32(lo_exp, hi_exp):
    """fp32 values on every exponent in [lo_exp, hi_exp]: all 11 top mantissa
    bits times low-bit patterns that straddle the e4m3 rounding points."""
    top = np.arange(1 << 11, dtype=np.uint32) << 12
    low = np.array([0, 1, 0x7FF, 0x800, 0x801, 0xFFF], dtype=np.uint32)
    mant = (top[:, None] | low[None, :]).ravel()
    out = []
    for e in range(lo_exp, hi_exp + 1):
        bits = (np.uint32(e + 127) << np.uint32(23)) | mant
        out.append(bits)
    bits = np.concatenate(out)
    v = bits.view(np.float32)
    return np.concatenate([v, -v])


def test_e4m3_vs_torch_in_range():
    v = _structured_f32(-24, 8)
    rng = np.random.default_rng(1)
    v = np.concatenate([v, rng.normal(0, 30, 1 << 20).astype(np.float32),
                        rng.uniform(-464, 464, 1 << 20).astype(np.float32)])
    v = v[np.abs(v) <= 464]
    got = oracle.e4m3_encode_array(v)
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    bad = np.nonzero(got != ref)[0]
    assert bad.size == 0, (v[bad[:5]], got[bad[:5]], ref[bad[:5]])


def test_e4m3_vs_nearest_code_search():
    """round to nearest code value, ties to the even mantissa, saturate"""
    tab = e4m3_table()
    codes = np.array(sorted(c for c in tab if c < 0x80), dtype=np.int64)
    vals = np.array([tab[c] for c in codes], dtype=np.float64)
    rng = np.random.default_rng(2)
    v = np.concatenate([rng.uniform(0, 500, 200000), rng.uniform(0, 0.05, 200000),
                        vals, (vals[1:] + vals[:-1]) / 2]).astype(np.float32)
    got = oracle.e4m3_encode_array(v)
    vv = v.astype(np.float64)
    d = np.abs(vv[:, None] - vals[None, :])
    dmin = d.min(axis=1, keepdims=True)
    cand = d == dmin
    even = (codes & 1) == 0
    pick = np.where(cand.sum(axis=1) > 1,
                    np.argmax(cand & even[None, :], axis=1), np.argmax(cand, axis=1))
    ref = codes[pick].astype(np.uint8)
    ref[vv >= 448.0] = 0x7E
    assert np.array_equal(got, ref)


def test_bf16_encode_vs_torch():
    rng = np.random.default_rng(3)
    base = rng.normal(0, 1, 1 << 18).astype(np.float32)
    bits = base.view(np.uint32) & np.uint32(0xFFFF0000)
    ties = (bits | np.uint32(0x8000)).view(np.float32)       # exact halfway cases
    near = (bits | np.uint32(0x7FFF)).view(np.float32)
    big = np.array([3.3895e38, 3.4e38, -3.4e38, 1e-40, -1e-45, 0.0, -0.0], np.float32)
    v = np.concatenate([base, ties, near, big])
    got = oracle.bf16_encode_array(v)
    ref = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got, ref)


# ---------------------------------------------------------------------------
# sigmoid
# ---------------------------------------------------------------------------

def test_sigmoid_matches_fp64_restatement():
    rng = np.random.default_rng(4)
    x = np.concatenate([rng.normal(0, 1, 20000), rng.uniform(-60, 60, 5000),
                        [0.0, 1e-30, -1e-30, 88.0, -88.0, -104.0, 17.0]]).astype(np.float32)
    got, hard = oracle.sigmoid_array(x)
    ref = np.array([sig_f32(v) for v in x], np.float32)
    ok = (got == ref) | (hard == 1)
    assert ok.all()
    assert oracle.sigmoid(0.0) == (F32(0.5), False)
    assert hard.sum() <= 2


def test_sigmoid_hard_flag_marks_midpoints():
    # choose x so that the fp64 sigmoid is within 2^-47 relative of an fp32
    # midpoint: invert the logistic at a midpoint m: x = log(m / (1 - m))
    a = F32(0.6)
    m = (float(a) + float(np.nextafter(a, F32(1)))) / 2
    x = F32(math.log(m / (1 - m)))
    v = 1 / (1 + math.exp(-float(x)))
    _, hard = oracle.sigmoid(float(x))
    assert hard == (abs(v - m) <= abs(v) * 2.0 ** -47)


# ---------------------------------------------------------------------------
# routing
# ---------------------------------------------------------------------------

ROUTE_CASES = [
    # (E, G, Kg, k)
    (16, 1, 1, 2),
    (16, 4, 2, 4),
    (32, 8, 3, 5),
    (12, 3, 2, 3),
]


@pytest.mark.parametrize("E,G,Kg,k", ROUTE_CASES)
@pytest.mark.parametrize("grid", [False, True])
def test_route_bruteforce(E, G, Kg, k, grid):
    rng = np.random.default_rng(E * 100 + G * 10 + k + grid)
    T = 48
    if grid:  # coarse values: many exact ties in keys and group scores
        logits = rng.choice([-1.0, 0.0, 1.0], size=(T, E)).astype(np.float32)
        bias = np.zeros(E, np.float32)
    else:
        logits = rng.normal(0, 1, (T, E)).astype(np.float32)
        bias = rng.uniform(-0.1, 0.1, E).astype(np.float32)
    for scale, renorm in [(1.0, True), (2.5, True), (1.7, False)]:
        idx, w, hard = oracle.route(logits, bias, G, Kg, k, scale, renorm)
        assert hard.sum() == 0
        for t in range(T):
            pick, ww = route_bruteforce(logits[t], bias, G, Kg, k, scale, renorm)
            assert list(idx[t]) == pick, (t, list(idx[t]), pick)
            assert np.array_equal(w[t], np.array(ww, np.float32))


def test_route_worked_examples():
    with open(os.path.join(GOLDEN, "route_worked_example.json")) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        lg = np.array([c["logits"]], np.float32)
        b = np.array(c["bias"], np.float32)
        idx, w, _ = oracle.route(lg, b, c["n_group"], c["topk_group"], c["topk"], 2.5, True)
        assert list(idx[0]) == c["topk_idx"]
        # closed form of the weights: scale * s_j / sum(s)
        s = [1 / (1 + math.exp(-c["logits"][e])) for e in c["topk_idx"]]
        for j in range(c["topk"]):
            assert w[0, j] == pytest.approx(2.5 * s[j] / sum(s), rel=1e-6)


def test_route_single_group_is_plain_topk():
    rng = np.random.default_rng(5)
    T, E, k = 256, 256, 8
    logits = rng.normal(0, 1, (T, E)).astype(np.float32)
    bias = rng.uniform(-0.1, 0.1, E).astype(np.float32)
    idx, w, hard = oracle.route(logits, bias, 1, 1, k, 1.0, False)
    s = 1 / (1 + np.exp(-logits.astype(np.float64)))
    keys = torch.from_numpy((s.astype(np.float32) + bias).astype(np.float32))
    ref = torch.topk(keys, k, dim=1, sorted=True).indices.numpy()
    ok = hard == 0
    assert np.array_equal(idx[ok], ref[ok])
    # no renorm, scale 1: weights are the plain fp32 sigmoid scores
    assert np.array_equal(w[ok], np.take_along_axis(s.astype(np.float32), idx, 1)[ok])


@pytest.mark.parametrize("E,G,Kg,k", [
    (16, 16, 2, 2),   # groups of one expert: no second key to score a group by
    (16, 3, 1, 2),    # E not a multiple of the group count
    (16, 4, 5, 2),    # more groups kept than there are
    (16, 4, 1, 5),    # more experts than the kept groups hold
    (16, 1, 1, 0),
])
def test_route_rejects_undefined_configurations(E, G, Kg, k):
    """the oracle refuses configurations the method leaves undefined (the
    group score is the sum of a group's two largest keys, so a group needs
    two experts) instead of reading past a group"""
    logits = np.zeros((3, E), np.float32)
    with pytest.raises(ValueError):
        oracle.route(logits, None, G, Kg, k, 1.0, True)


def test_route_two_expert_groups_brute_force():
    """the smallest groups the method defines (two experts: the group score
    is the sum of both keys) against exhaustive enumeration of group subsets"""
    import itertools
    rng = np.random.default_rng(17)
    E, G, Kg, k = 8, 4, 2, 3
    logits = rng.normal(0, 1, (64, E)).astype(np.float32)
    idx, _, hard = oracle.route(logits, None, G, Kg, k, 1.0, False)
    s = (1 / (1 + np.exp(-logits.astype(np.float64)))).astype(np.float32)
    for t in range(64):
        if hard[t]:
            continue
        gscore = [np.float32(s[t, 2 * g]) + np.float32(s[t, 2 * g + 1]) for g in range(G)]
        best = max(itertools.combinations(range(G), Kg),
                   key=lambda c: (sorted((gscore[g] for g in c), reverse=True),
                                  [-g for g in c]))
        allowed = [e for e in range(E) if e // 2 in best]
        want = sorted(allowed, key=lambda e: (-s[t, e], e))[:k]
        assert list(idx[t]) == want


def test_route_invariants_v3_shape():
    cfg = CONFIGS["v3"].scaled(512)
    wl = Workload(cfg)
    idx, w, hard = oracle.route(wl.logits, wl.bias, cfg.n_group, cfg.topk_group,
                                cfg.topk, cfg.routed_scale, cfg.renorm)
    gs = cfg.E // cfg.n_group
    for t in range(cfg.T):
        assert len(set(idx[t])) == cfg.topk
        assert len(set(int(e) // gs for e in idx[t])) <= cfg.topk_group
        assert (w[t] > 0).all()
        assert abs(float(w[t].astype(np.float64).sum()) - cfg.routed_scale) <= \
            cfg.topk * 4 * cfg.routed_scale * 2.0 ** -24
    # selection order: keys non-increasing along j
    s = 1 / (1 + np.exp(-wl.logits.numpy().astype(np.float64)))
    keys = s.astype(np.float32) + wl.bias.numpy()
    kk = np.take_along_axis(keys, idx, 1)
    assert (np.diff(kk, axis=1) <= 0).all()


# ---------------------------------------------------------------------------
# layout
# ---------------------------------------------------------------------------

def layout_by_sort(topk_idx, E, P, R, phys_of=None, n_rep=None):
    """slot of (t,j) = position of (p, t, j) in the sorted list of pairs"""
    T, k = topk_idx.shape
    pairs = []
    for t in range(T):
        for j in range(k):
            e = int(topk_idx[t, j])
            p = e if phys_of is None else int(phys_of[e, t % int(n_rep[e])])
            pairs.append((p, t, j))
    order = sorted(pairs)
    slot = np.zeros((T, k), np.int32)
    for pos, (p, t, j) in enumerate(order):
        slot[t, j] = pos
    cnt = np.bincount([p for p, _, _ in pairs], minlength=P)
    return slot, cnt


def check_layout_invariants(lay, topk_idx, E, P, R, phys_of=None, n_rep=None):
    T, k = topk_idx.shape
    epr = P // R
    cnt = lay["cnt_expert"]
    assert cnt.sum() == T * k
    assert np.array_equal(lay["expert_off"], np.concatenate([[0], np.cumsum(cnt)]))
    slot = lay["slot"].ravel()
    assert np.array_equal(np.sort(slot), np.arange(T * k))
    src = lay["src"]
    assert np.array_equal(src[slot], np.arange(T * k))
    tok_of_row = src // k
    for p in range(P):
        rows = tok_of_row[lay["expert_off"][p]:lay["expert_off"][p + 1]]
        assert (np.diff(rows) >= 0).all()
    for r in range(R):
        assert lay["rows_rank"][r] == cnt[r * epr:(r + 1) * epr].sum()
        assert lay["rank_off"][r] == lay["expert_off"][r * epr]
    phys = np.zeros((T, k), np.int64)
    for t in range(T):
        for j in range(k):
            e = int(topk_idx[t, j])
            phys[t, j] = e if phys_of is None else int(phys_of[e, t % int(n_rep[e])])
    ranks = phys // epr
    in_rank = np.zeros((T, R), np.uint8)
    for t in range(T):
        in_rank[t, np.unique(ranks[t])] = 1
    assert np.array_equal(lay["in_rank"], in_rank)
    assert np.array_equal(lay["tok_rank"], in_rank.sum(0))
    # each receive row holds the expert it was counted for
    row_expert = np.repeat(np.arange(P), cnt)
    assert np.array_equal(row_expert[slot], phys.ravel())


@pytest.mark.parametrize("name", ["tiny", "ds16b", "v3", "skew"])
def test_layout_vs_sort_and_invariants(name):
    cfg = CONFIGS[name].scaled(96)
    wl = Workload(cfg)
    idx, _, _ = oracle.route(wl.logits, wl.bias, cfg.n_group, cfg.topk_group,
                             cfg.topk, cfg.routed_scale, cfg.renorm)
    po = None if wl.phys_of is None else wl.phys_of.numpy()
    nr = None if wl.n_rep is None else wl.n_rep.numpy()
    lay = oracle.layout(idx, cfg.E, cfg.n_phys, cfg.R, po, nr)
    assert lay["status"] == 0
    slot, cnt = layout_by_sort(idx, cfg.E, cfg.n_phys, cfg.R, po, nr)
    assert np.array_equal(lay["slot"], slot)
    assert np.array_equal(lay["cnt_expert"], cnt)
    check_layout_invariants(lay, idx, cfg.E, cfg.n_phys, cfg.R, po, nr)
    if po is not None:  # replicas of a logical expert sum to its logical count
        logical = np.bincount(idx.ravel(), minlength=cfg.E)
        for e in range(cfg.E):
            reps = po[e, :nr[e]]
            assert lay["cnt_expert"][reps].sum() == logical[e]


def test_layout_invalid_ids_flagged():
    idx = np.array([[0, 3], [5, 1], [-1, 2]], np.int32)
    lay = oracle.layout(idx, 4, 4, 2)
    assert lay["status"] & oracle.BAD_EXPERT
    assert lay["slot"][1, 0] == -1 and lay["slot"][2, 0] == -1
    assert lay["cnt_expert"].sum() == 4
    po = np.array([[0, 1], [2, -1], [3, -1], [9, -1]], np.int32)
    nr = np.array([2, 1, 1, 1], np.int32)
    lay = oracle.layout(np.array([[3, 0]], np.int32), 4, 4, 2, po, nr)
    assert lay["status"] & oracle.BAD_REPLICA and lay["slot"][0, 0] == -1


def test_layout_pages_counting_facts():
    with open(os.path.join(GOLDEN, "perplexity_counting.json")) as f:
        g = json.load(f)
    # batch of 2 tokens (batch 1, query length 2) reaches at most 2*8 experts
    a = g["activated_experts_batch1"]
    cfg = CONFIGS["v3"]
    assert cfg.topk == a["topk"] and cfg.E == a["experts"] and cfg.R == a["ep"]
    for seed in range(20):
        wl = Workload(cfg.scaled(a["tokens"]), seed=seed)
        idx, _, _ = oracle.route(wl.logits, wl.bias, cfg.n_group, cfg.topk_group,
                                 cfg.topk, cfg.routed_scale, cfg.renorm)
        lay = oracle.layout(idx, cfg.E, cfg.E, cfg.R)
        active = int((lay["cnt_expert"] > 0).sum())
        assert active <= a["max_activated_experts"]
        # mean activated experts per GPU: active / EP, = 2 when all 16 differ
        assert active / a["ep"] <= a["mean_activated_per_gpu"]
        if active == a["tokens"] * a["topk"]:
            assert active / a["ep"] == a["mean_activated_per_gpu"]
    # a large batch activates every expert: 256 / 8 = 32 per GPU (unbiased
    # gate, as in the page's setting; a selection bias can starve experts)
    wl = Workload(cfg.scaled(1024))
    idx, _, _ = oracle.route(wl.logits, None, cfg.n_group, cfg.topk_group,
                             cfg.topk, cfg.routed_scale, cfg.renorm)
    lay = oracle.layout(idx, cfg.E, cfg.E, cfg.R)
    per_rank = (lay["cnt_expert"] > 0).reshape(cfg.R, -1).sum(1)
    assert (per_rank == a["all_activated_per_gpu"]).all()
    # balanced routing: m = 128*2*8*128/256 = 1024 tokens per expert
    b = g["groupgemm_tokens_per_expert"]
    T = b["batch_per_gpu"] * b["query_len"] * b["dp"]
    k, E = b["topk"], b["experts"]
    t = np.arange(T)[:, None]
    j = np.arange(k)[None, :]
    balanced = ((t * k + j) % E).astype(np.int32)   # round-robin assignment
    lay = oracle.layout(balanced, E, E, 128)
    assert (lay["cnt_expert"] == b["tokens_per_expert"]).all()
    c = g["ep128_experts_per_gpu"]
    assert c["experts"] // c["ep"] == c["experts_per_gpu"]
    assert (lay["rows_rank"] == c["experts_per_gpu"] * b["tokens_per_expert"]).all()


# ---------------------------------------------------------------------------
# dispatch (quantise) and combine
# ---------------------------------------------------------------------------

def _bf16_rows(rng, T, H, scale=1.0):
    return torch.from_numpy(rng.normal(0, scale, (T, H)).astype(np.float32)).to(torch.bfloat16)


def test_quantize_scale_identity_and_error_bound():
    rng = np.random.default_rng(6)
    x = _bf16_rows(rng, 16, 1024, 3.0)
    x[3, 128:256] = 0.0                  # all-zero block
    x[4, 0:128] = -0.0
    x[5, 256:384] = torch.tensor(1e-38, dtype=torch.bfloat16)  # tiny amax
    for t in range(16):
        q, sc = oracle.quantize_row(x[t])
        xf = x[t].float().numpy().reshape(-1, 128)
        amax = np.abs(xf).max(1).astype(np.float32)
        assert np.array_equal(sc, (amax / F32(448.0)).astype(np.float32))
        deq = torch.from_numpy(q).view(torch.float8_e4m3fn).float().numpy().reshape(-1, 128)
        for b in range(xf.shape[0]):
            if amax[b] == 0:
                assert (q.reshape(-1, 128)[b] == 0).all() and sc[b] == 0
                continue
            err = np.abs(deq[b] * np.float64(sc[b]) - xf[b])
            bound = np.maximum(np.abs(xf[b]) * 2.0 ** -4, 2.0 ** -10 * np.float64(sc[b]))
            assert (err <= bound * (1 + 2.0 ** -20)).all()
            # the block maximum maps to (or saturates at) 448
            assert np.abs(deq[b]).max() == 448.0
        # q equals a direct RN conversion of fp32(x / scale) (torch, in range)
        with np.errstate(divide="ignore", invalid="ignore"):
            ratio = (xf / sc[:, None]).astype(np.float32)
        nz = sc > 0
        ref = torch.from_numpy(ratio[nz]).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
        assert np.array_equal(q.reshape(-1, 128)[nz], ref)


def test_dispatch_bf16_is_bitwise_permutation():
    rng = np.random.default_rng(7)
    T, H, k = 40, 256, 3
    x = _bf16_rows(rng, T, H)
    slot = rng.permutation(T * k).astype(np.int32).reshape(T, k)
    rx, _ = oracle.dispatch(x, slot, fp8=False)
    xb = x.view(torch.int16).numpy().view(np.uint16)
    for t in range(T):
        for j in range(k):
            assert np.array_equal(rx[slot[t, j]], xb[t])


def test_combine_vs_fp64_sum():
    rng = np.random.default_rng(8)
    T, H, k = 24, 384, 6
    y = _bf16_rows(rng, T * k, H)
    slot = rng.permutation(T * k).astype(np.int32).reshape(T, k)
    w = rng.uniform(0.01, 1.0, (T, k)).astype(np.float32)
    out = oracle.combine(y, slot, w)
    yf = y.float().numpy().astype(np.float64)
    ref = np.einsum("tj,tjh->th", w.astype(np.float64), yf[slot])
    got = torch.from_numpy(out.view(np.int16)).view(torch.bfloat16).float().numpy()
    mag = np.einsum("tj,tjh->th", w.astype(np.float64), np.abs(yf[slot]))
    assert (np.abs(got - ref) <= 2.0 ** -8 * np.abs(ref) + k * 2.0 ** -23 * mag + 1e-30).all()
    # a dropped term or a wrong weight would move results by O(|w y|)
    w2 = w.copy()
    w2[:, -1] = 0
    out2 = oracle.combine(y, slot, w2)
    assert not np.array_equal(out, out2)


def test_identity_expert_round_trip():
    """dispatch -> dequantised identity experts -> combine recovers x"""
    cfg = CONFIGS["ds16b"].scaled(64)
    wl = Workload(cfg)
    idx, w, _ = oracle.route(wl.logits, wl.bias, 1, 1, cfg.topk, 1.0, True)
    lay = oracle.layout(idx, cfg.E, cfg.E, cfg.R)
    rx, rs = oracle.dispatch(wl.x, lay["slot"], fp8=True)
    deq = torch.from_numpy(rx).view(torch.float8_e4m3fn).float() * \
        torch.from_numpy(np.repeat(rs, 128, axis=1))
    y = deq.to(torch.bfloat16)
    out = oracle.combine(y, lay["slot"], w)
    got = torch.from_numpy(out.view(np.int16)).view(torch.bfloat16).float().numpy()
    x = wl.x.float().numpy()
    sc = np.repeat(np.abs(x).reshape(cfg.T, -1, 128).max(2) / 448.0, 128, axis=1)
    bound = (2.0 ** -4 + 2.0 ** -7) * np.abs(x) + 2.0 ** -9 * sc + 1e-30
    assert (np.abs(got - x) <= bound).all()
    # bf16 mode with identity experts: y rows are x itself
    rxb, _ = oracle.dispatch(wl.x, lay["slot"], fp8=False)
    yb = torch.from_numpy(rxb.view(np.int16)).view(torch.bfloat16)
    outb = oracle.combine(yb, lay["slot"], w)
    gotb = torch.from_numpy(outb.view(np.int16)).view(torch.bfloat16).float().numpy()
    assert (np.abs(gotb - x) <= 2.0 ** -8 * np.abs(x) + 1e-30).all()


# ---------------------------------------------------------------------------
# backward
# ---------------------------------------------------------------------------

def _bf16f(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).double().numpy()


def test_dispatch_backward_is_the_adjoint_of_dispatch():
    """<dispatch(x), r> == <x, dispatch_backward(r)> for the bf16 permutation
    (up to the bf16 rounding of the backward sum)"""
    rng = np.random.default_rng(31)
    T, H, k = 50, 256, 4
    x = _bf16_rows(rng, T, H)
    r = _bf16_rows(rng, T * k, H)
    slot = rng.permutation(T * k).astype(np.int32).reshape(T, k)
    rx, _ = oracle.dispatch(x, slot, fp8=False)
    lhs = float((_bf16f(rx) * r.double().numpy()).sum())
    gx = oracle.dispatch_backward(r, slot)
    rhs = float((x.double().numpy() * _bf16f(gx)).sum())
    mag = float((np.abs(x.double().numpy()) * np.abs(_bf16f(gx))).sum())
    assert abs(lhs - rhs) <= 2.0 ** -8 * mag
    # exact restatement of the sum (fp64, then the bf16 rounding bound)
    ref = r.double().numpy()[slot].sum(axis=1)
    assert (np.abs(_bf16f(gx) - ref) <= 2.0 ** -8 * np.abs(ref) + k * 2.0 ** -23 *
            np.abs(r.double().numpy()[slot]).sum(axis=1) + 1e-30).all()


def test_combine_backward_gradients():
    rng = np.random.default_rng(32)
    T, H, k = 40, 384, 6
    y = _bf16_rows(rng, T * k, H)
    g = _bf16_rows(rng, T, H)
    slot = rng.permutation(T * k).astype(np.int32).reshape(T, k)
    w = rng.uniform(0.05, 1.5, (T, k)).astype(np.float32)
    gy, gw = oracle.combine_backward(g, y, slot, w)
    gf, yf = g.double().numpy(), y.double().numpy()
    # grad_w: derivative of sum_h g[t,h] * out[t,h] wrt w[t,j] is <g[t], y[slot]>
    ref_w = np.einsum("th,tjh->tj", gf, yf[slot])
    assert np.allclose(gw, ref_w, rtol=1e-6, atol=1e-6)
    # grad_y rows: w * g[t], one fp32 product rounded to bf16
    for t in range(T):
        for j in range(k):
            exp = torch.from_numpy((w[t, j] * g[t].float().numpy()).astype(np.float32)).to(
                torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
            assert np.array_equal(gy[slot[t, j]], exp)
    # adjoint: <combine(y), g> == <y, grad_y> (before bf16 rounding of either side)
    out = oracle.combine(y, slot, w)
    lhs = float((_bf16f(out) * gf).sum())
    rhs = float((yf * _bf16f(gy)).sum())
    assert abs(lhs - rhs) <= 2.0 ** -7 * float((np.abs(_bf16f(out)) * np.abs(gf)).sum())
    # a finite-difference check of one weight's gradient
    t, j, eps = 3, 2, 1e-3
    w2 = w.copy()
    w2[t, j] += eps
    f = lambda ww: (np.einsum("tj,tjh->th", ww.astype(np.float64), yf[slot]) * gf).sum()
    delta = float(w2[t, j]) - float(w[t, j])  # the step actually stored in fp32
    assert (f(w2) - f(w)) / delta == pytest.approx(gw[t, j], rel=1e-6, abs=1e-6)


@pytest.mark.parametrize("align", [1, 4, 64, 128])
def test_layout_row_alignment(align):
    """padded expert starts: multiples of the row tile, the same rows per
    expert in the same order, padding rows marked -1"""
    cfg = CONFIGS["skew"].scaled(300)
    wl = Workload(cfg, seed=5)
    idx, _, _ = oracle.route(wl.logits, wl.bias, cfg.n_group, cfg.topk_group, cfg.topk,
                             cfg.routed_scale, cfg.renorm)
    po, nr = wl.phys_of.numpy(), wl.n_rep.numpy()
    base = oracle.layout(idx, cfg.E, cfg.n_phys, cfg.R, po, nr)
    lay = oracle.layout(idx, cfg.E, cfg.n_phys, cfg.R, po, nr, row_align=align)
    P = cfg.n_phys
    cnt = lay["cnt_expert"]
    assert np.array_equal(cnt, base["cnt_expert"])
    assert np.array_equal(lay["tok_rank"], base["tok_rank"])
    assert np.array_equal(lay["in_rank"], base["in_rank"])
    off = lay["expert_off"]
    assert (off % align == 0).all()
    assert np.array_equal(np.diff(off), -(-cnt // align) * align)
    # pair (t, j) keeps its rank inside its expert
    phys = np.searchsorted(base["expert_off"], base["slot"], side="right") - 1
    assert np.array_equal(lay["slot"] - off[phys], base["slot"] - base["expert_off"][phys])
    src = lay["src"]
    assert src.size == off[P]
    assert np.array_equal(src[lay["slot"].ravel()], np.arange(cfg.T * cfg.topk))
    assert (src >= 0).sum() == cfg.T * cfg.topk
    epr = P // cfg.R
    assert np.array_equal(lay["rank_off"], off[::epr])
    assert np.array_equal(lay["rows_rank"], np.diff(off[::epr]))
    if align == 1:
        for n in ("expert_off", "slot", "src", "rows_rank", "rank_off"):
            assert np.array_equal(lay[n], base[n])


def _padded_layout_restatement(idx, E, R, align):
    """slots by a stable sort of the pairs by expert (pairs in (t, j) order),
    expert starts rounded up to the row tile"""
    T, k = idx.shape
    flat = idx.reshape(-1)
    order = np.argsort(flat, kind="stable")
    cnt = np.bincount(flat, minlength=E)
    padded = -(-cnt // align) * align
    off = np.concatenate([[0], np.cumsum(padded)])
    first_in_sorted = np.concatenate([[0], np.cumsum(cnt)])
    slot = np.empty(T * k, np.int64)
    for pos, pair in enumerate(order):
        e = flat[pair]
        slot[pair] = off[e] + (pos - first_in_sorted[e])
    epr = E // R
    return cnt, off, slot.reshape(T, k), off[::epr]


@settings(max_examples=60, deadline=None)
@given(T=st.integers(1, 40), k=st.integers(1, 4), epr=st.integers(1, 4), R=st.integers(1, 4),
       align=st.sampled_from([1, 2, 3, 8, 16]), seed=st.integers(0, 2 ** 31 - 1))
def test_padded_layout_vs_sort_restatement(T, k, epr, R, align, seed):
    E = epr * R
    if k > E:
        k = E
    rng = np.random.default_rng(seed)
    idx = np.stack([rng.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32)
    lay = oracle.layout(idx, E, E, R, row_align=align)
    cnt, off, slot, rank_off = _padded_layout_restatement(idx, E, R, align)
    assert np.array_equal(lay["cnt_expert"], cnt)
    assert np.array_equal(lay["expert_off"], off)
    assert np.array_equal(lay["slot"], slot)
    assert np.array_equal(lay["rank_off"], rank_off)
    src = np.full(off[-1], -1)
    src[slot.reshape(-1)] = np.arange(T * k)
    assert np.array_equal(lay["src"], src)
