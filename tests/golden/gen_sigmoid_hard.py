#!/usr/bin/env python
"""Writes tests/golden/sigmoid_hard_inputs.txt: every fp32 input whose
sigmoid, evaluated in fp64, lies within 2^-47 (relative) of an fp32 rounding
midpoint, so that fp64 alone cannot be trusted to round it (the routing's
reading of the sigmoid: the exact value rounded once to fp32).

It calls the oracle only: ``oracle.sigmoid_hard_scan`` over all 2^32 bit
patterns (NaN skipped), in ranges on the host's cores.

    python tests/golden/gen_sigmoid_hard.py
"""

import os
import sys
from concurrent.futures import ThreadPoolExecutor

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402

OUT = os.path.join(os.path.dirname(os.path.abspath(__file__)), "sigmoid_hard_inputs.txt")
CHUNK = 1 << 24


def main():
    starts = range(0, 1 << 32, CHUNK)
    with ThreadPoolExecutor(max_workers=os.cpu_count() or 1) as ex:
        parts = list(ex.map(lambda s: oracle.sigmoid_hard_scan(s, CHUNK), starts))
    bits = np.concatenate(parts)
    with open(OUT, "w") as f:
        f.write("# fp32 inputs x (bit patterns, hex) whose sigmoid 1/(1+e^-x), evaluated in\n")
        f.write("# fp64, lies within 2^-47 (relative) of an fp32 rounding midpoint; written by\n")
        f.write("# tests/golden/gen_sigmoid_hard.py from oracle.sigmoid_hard_scan over all\n")
        f.write(f"# 2^32 patterns.  {bits.size} inputs.\n")
        for b in bits:
            f.write("%08x\n" % int(b))
    print(OUT, bits.size)


if __name__ == "__main__":
    main()
