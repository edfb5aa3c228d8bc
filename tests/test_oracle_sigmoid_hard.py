"""The routing sigmoid near fp32 rounding midpoints.

Reading of the sigmoid: the exact 1 / (1 + e^-x) rounded once to fp32.  For
most inputs an fp64 evaluation decides the rounding; tests/golden/
sigmoid_hard_inputs.txt lists every fp32 input (all 2^32 patterns scanned by
the oracle) whose fp64 value lies within 2^-47 of a midpoint, where the
oracle decides again in quad precision.  Here each listed input is checked
against an independent 80-digit decimal evaluation rounded to fp32 by exact
comparison, and a random sample checks that the list misses no input that
numpy's fp64 evaluation also finds near a midpoint.
"""

import os
from decimal import Decimal, getcontext

import numpy as np

import oracle

HERE = os.path.dirname(os.path.abspath(__file__))


def hard_inputs() -> np.ndarray:
    bits = [int(ln, 16) for ln in open(os.path.join(HERE, "golden", "sigmoid_hard_inputs.txt"))
            if ln.strip() and not ln.startswith("#")]
    return np.array(bits, np.uint32).view(np.float32)


def exact_sigmoid(x: np.float32) -> Decimal:
    getcontext().prec = 80
    return Decimal(1) / (Decimal(1) + (-Decimal(float(x))).exp())


def round_to_fp32(v: Decimal):
    """the fp32 nearest to v (ties to even), and v's distance from the
    midpoint between it and its neighbour on v's side, relative to v"""
    c = np.float32(float(v))
    up, dn = np.float32(np.inf), np.float32(-np.inf)
    cands = [np.nextafter(c, dn), c, np.nextafter(c, up)]
    best = min(cands, key=lambda f: (abs(Decimal(float(f)) - v),
                                     int(np.array(f, np.float32).view(np.uint32)) & 1))
    nb = np.nextafter(best, up if Decimal(float(best)) < v else dn)
    mid = (Decimal(float(best)) + Decimal(float(nb))) / 2
    return best, abs(v - mid) / v


def test_every_hard_input_is_correctly_rounded():
    x = hard_inputs()
    assert 500 <= x.size <= 5000
    got, hard = oracle.sigmoid_array(x)
    assert hard.all()  # the oracle flags each listed input itself
    fp64_wrong = 0
    for xi, gi in zip(x, got):
        want, rel = round_to_fp32(exact_sigmoid(xi))
        assert np.array_equal(np.float32(gi).view(np.uint32), np.float32(want).view(np.uint32)), \
            (float(xi), float(gi), float(want))
        # far enough from the midpoint for quad precision (2^-112) to decide
        assert rel > Decimal(2) ** -100, float(xi)
        v64 = np.float32(1.0 / (1.0 + np.exp(-np.float64(xi))))
        fp64_wrong += int(v64 != want)
    # rounding the fp64 value alone goes wrong on some of them: the quad
    # step is what the list exists for
    assert fp64_wrong > 0


def test_list_contains_the_inputs_near_zero():
    """for tiny x, sigmoid(x) = 1/2 + x/4 - x^3/48 + ..., so x/4 on a
    midpoint of the fp32 grid around 1/2 puts the value a hair from it: such
    inputs must be in the list"""
    x = set(hard_inputs().view(np.uint32).tolist())
    for xv in (np.float32(2.0 ** -23 * 3), np.float32(-(2.0 ** -24) * 5)):
        assert int(np.array(xv, np.float32).view(np.uint32)) in x, float(xv)


def test_random_sample_finds_no_unlisted_hard_input():
    rng = np.random.default_rng(7)
    listed = set(hard_inputs().view(np.uint32).tolist())
    xs = np.concatenate([rng.uniform(-110, 40, 1 << 20),
                         rng.normal(0, 2.0 ** -18, 1 << 18)]).astype(np.float32)
    v = 1.0 / (1.0 + np.exp(-xs.astype(np.float64)))
    f = v.astype(np.float32)
    other = np.where(v >= f, np.nextafter(f, np.float32(np.inf)), np.nextafter(f, np.float32(-np.inf)))
    mid = 0.5 * (f.astype(np.float64) + other.astype(np.float64))
    near = np.abs(v - mid) <= np.ldexp(np.abs(v), -47)
    for b in xs[near].view(np.uint32):
        assert int(b) in listed
