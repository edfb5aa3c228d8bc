"""Pins for the oracle's expert activation (SiLU(gate) * up, then the 1x128
FP8 quantiser), each against something other than the oracle itself.

SiLU: every bf16 input, evaluated with Python's ``decimal`` at 60 digits and
rounded to bf16 by exact rational arithmetic, plus its special values.
Product and rounding: numpy float32 products and an integer bf16 rounding.
Row selection: sentinel rows that the per-expert counts leave out.
"""

import math
import struct
from decimal import Decimal, localcontext
from fractions import Fraction

import numpy as np
import pytest

import oracle
from gen import CONFIGS, Workload


def bf16_value(bits: int) -> float:
    return struct.unpack("<f", struct.pack("<I", (int(bits) & 0xFFFF) << 16))[0]


def round_bf16_exact(v: Fraction, negative: bool) -> int:
    """bf16 bits of the exact rational v, to nearest, ties to even (an exact
    tie never occurs for v = silu(x), x != 0, which is transcendental)."""
    sign = 0x8000 if negative else 0
    a = abs(v)
    if a == 0:
        return sign
    e = a.numerator.bit_length() - a.denominator.bit_length()
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    q = Fraction(2) ** (max(e, -126) - 7)   # bf16 step at this magnitude
    n = a / q
    fl = n.numerator // n.denominator
    rem = n - fl
    r = fl + (1 if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2) else 0)
    val = r * q
    if val >= 2 ** 128:
        return sign | 0x7F80
    bits = struct.unpack("<I", struct.pack("<f", float(val)))[0]
    return sign | (bits >> 16)


def silu_reference(bits: int) -> int:
    """bf16 bits of silu(x) for bf16 bits x, from a 60-digit evaluation."""
    x = bf16_value(bits)
    if math.isnan(x):
        return -1                       # any NaN
    if math.isinf(x):
        return 0x7F80 if x > 0 else 0x8000
    if x == 0:
        return bits                     # silu(+-0) = +-0
    if x > 1000:                        # x (1 - e^-x ...): e^-1000 < 2^-1400
        return bits
    if x < -1000:                       # |x e^x| < 2^-1400: rounds to -0
        return 0x8000
    with localcontext() as ctx:
        ctx.prec = 60
        d = Decimal(x)                  # exact
        v = d / (1 + (-d).exp())
    return round_bf16_exact(Fraction(v), x < 0)


def bf16_round_f32(a: np.ndarray) -> np.ndarray:
    """bf16 bits of float32 values, to nearest, ties to even, by integer
    arithmetic on the float32 pattern (NaN stays NaN)."""
    u = a.astype(np.float32).view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + lsb) >> 16).astype(np.uint16)
    nan = np.isnan(a)
    r[nan] = ((u[nan] >> 16) | 0x40).astype(np.uint16)
    return r


@pytest.fixture(scope="module")
def silu_table():
    g = np.arange(65536, dtype=np.uint16)
    s, hard = oracle.silu_bf16_array(g)
    return s, hard


def test_silu_every_bf16_input_vs_60_digit_evaluation(silu_table):
    s, hard = silu_table
    assert hard.sum() == 0, "an input lies too close to a rounding midpoint"
    bad = []
    for b in range(65536):
        ref = silu_reference(b)
        got = int(s[b])
        if ref < 0:
            ok = math.isnan(bf16_value(got))
        else:
            ok = got == ref
        if not ok:
            bad.append((hex(b), hex(got), hex(ref)))
    assert not bad, bad[:10]


def test_silu_special_values(silu_table):
    s, _ = silu_table
    assert s[0x0000] == 0x0000 and s[0x8000] == 0x8000          # +-0
    assert s[0x7F80] == 0x7F80 and s[0xFF80] == 0x8000          # +inf, -inf -> -0
    assert math.isnan(bf16_value(s[0x7FC0]))
    assert s[0x3F80] == 0x3F3B                                  # silu(1) = 0.7310...
    assert bf16_value(s[0x3F80]) == 0.73046875
    # large positive x: silu(x) = x; large negative: -0
    for x in (16.0, 100.0, 3.0e38):
        b = struct.unpack("<I", struct.pack("<f", x))[0] >> 16
        assert s[b] == b
    assert s[0xC3C8] == 0x8000                                  # silu(-400) = -0
    # smallest subnormals: silu(x) lies just above x/2 (ties round up)
    assert s[0x0001] == 0x0001 and s[0x8001] == 0x8000
    assert s[0x0003] == 0x0002 and s[0x8003] == 0x8001


def test_silu_reflection_identity(silu_table):
    """silu(x) - silu(-x) = x exactly in the reals: with each side rounded
    once to bf16, the identity holds within the two roundings."""
    s, _ = silu_table
    b = np.arange(0x0080, 0x4300, dtype=np.uint32)        # 2^-126 <= x < 128
    xp = np.array([bf16_value(v) for v in b])
    sp = np.array([bf16_value(s[v]) for v in b])
    sn = np.array([bf16_value(s[v | 0x8000]) for v in b])
    ulp = lambda v: np.maximum(np.abs(v), 2.0 ** -126) * 2.0 ** -8  # noqa: E731
    assert np.all(np.abs((sp - sn) - xp) <= ulp(sp) + ulp(sn))


def activation_restatement(gate_up_bits: np.ndarray, silu_bits: np.ndarray) -> np.ndarray:
    """h bits = bf16(fp32(silu_bf16(gate) * up)) with numpy float32 products."""
    I = gate_up_bits.shape[1] // 2
    g, u = gate_up_bits[:, :I], gate_up_bits[:, I:]
    s = (silu_bits[g].astype(np.uint32) << 16).view(np.float32)
    uf = (u.astype(np.uint32) << 16).view(np.float32)
    with np.errstate(over="ignore", invalid="ignore"):
        return bf16_round_f32(s * uf)


def random_gate_up(rows, I, seed):
    rng = np.random.default_rng(seed)
    x = (rng.standard_normal((rows, 2 * I)) * 2.0).astype(np.float32)
    bits = bf16_round_f32(x)
    # salt with special and extreme values
    special = np.array([0x0000, 0x8000, 0x7F80, 0xFF80, 0x0001, 0x8001, 0x7F7F, 0xFF7F,
                        0x0080, 0x3F80, 0xC2C8, 0x42C8], np.uint16)
    pos = rng.integers(0, bits.size, 64)
    bits.reshape(-1)[pos] = special[rng.integers(0, special.size, 64)]
    return bits


def test_activation_bf16_vs_float32_restatement(silu_table):
    s, _ = silu_table
    gu = random_gate_up(40, 256, 1)
    h, _ = oracle.silu_mul_quant(gu, fp8=False)
    ref = activation_restatement(gu, s)
    hf = (h.astype(np.uint32) << 16).view(np.float32)
    rf = (ref.astype(np.uint32) << 16).view(np.float32)
    both_nan = np.isnan(hf) & np.isnan(rf)
    assert np.array_equal(h[~both_nan], ref[~both_nan])
    assert np.array_equal(np.isnan(hf), np.isnan(rf))
    # up = 1 leaves silu itself
    gu2 = gu.copy()
    gu2[:, 256:] = 0x3F80
    h1, _ = oracle.silu_mul_quant(gu2, fp8=False)
    assert np.array_equal(h1, s[gu2[:, :256]])


def test_activation_fp8_is_the_quantiser_of_h(silu_table):
    s, _ = silu_table
    gu = random_gate_up(24, 512, 2)
    gu[gu == 0x7F80] = 0x3F80           # keep the blocks finite here
    gu[gu == 0xFF80] = 0xBF80
    q, sc = oracle.silu_mul_quant(gu, fp8=True)
    h = activation_restatement(gu, s)
    for r in range(gu.shape[0]):
        q_ref, sc_ref = oracle.quantize_row(h[r])
        assert np.array_equal(q[r], q_ref)
        assert np.array_equal(sc[r], sc_ref)
    # the scale is amax(|h|) / 448 per 128-element block
    hf = (h.astype(np.uint32) << 16).view(np.float32).reshape(gu.shape[0], -1, 128)
    amax = np.nanmax(np.abs(hf), axis=2)
    assert np.array_equal(sc, (amax / np.float32(448.0)).astype(np.float32))


def test_activation_processes_exactly_the_counted_rows():
    cfg = CONFIGS["tiny"].scaled(64)
    wl = Workload(cfg, seed=3)
    idx, _, _ = oracle.route(wl.logits, wl.bias, cfg.n_group, cfg.topk_group, cfg.topk,
                             cfg.routed_scale, cfg.renorm)
    lay = oracle.layout(idx, cfg.E, cfg.n_phys, cfg.R, row_align=8)
    n_rows = int(lay["expert_off"][-1]) + 5          # unused tail rows too
    I = 128
    gu = random_gate_up(n_rows, I, 4)
    sentinel_q = np.full((n_rows, I), 0xA5, np.uint8)
    sentinel_s = np.full((n_rows, 1), -7.0, np.float32)
    q, sc = oracle.silu_mul_quant(gu, True, lay["expert_off"], lay["cnt_expert"],
                                  sentinel_q.copy(), sentinel_s.copy())
    valid = np.zeros(n_rows, bool)
    for p in range(cfg.n_phys):
        o = lay["expert_off"][p]
        valid[o:o + lay["cnt_expert"][p]] = True
    assert valid.sum() == cfg.T * cfg.topk
    src = np.concatenate([lay["src"], np.full(5, -1, np.int32)])
    assert np.array_equal(valid, src >= 0)
    assert np.all(q[~valid] == 0xA5) and np.all(sc[~valid] == -7.0)
    full_q, full_s = oracle.silu_mul_quant(gu, True)
    assert np.array_equal(q[valid], full_q[valid]) and np.array_equal(sc[valid], full_s[valid])
