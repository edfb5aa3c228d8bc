"""The expert activation's SiLU table is generated on the host at build time
(csrc/gen_silu_table.c), one entry per bf16 gate pattern; every entry must
equal the oracle's correctly rounded SiLU of the same gate (NaN gates: a NaN
pattern on both sides)."""

import numpy as np

import oracle
from combine_ep_route_02_b200 import build as B


def is_nan_bf16(b):
    return ((b & 0x7F80) == 0x7F80) & ((b & 0x007F) != 0)


def test_silu_table_equals_oracle(tmp_path):
    B.generate_tables(str(tmp_path))
    text = (tmp_path / "silu_table.inc").read_text()
    got = np.array([int(v, 16) for v in text.replace("\n", " ").split(",") if v.strip()],
                   dtype=np.uint16)
    assert got.size == 65536
    gate = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref, hard = oracle.silu_bf16_array(gate)
    assert hard.sum() == 0
    nan = is_nan_bf16(gate)
    assert nan.sum() == 2 * 127
    assert np.array_equal(got[~nan], ref[~nan])
    assert is_nan_bf16(got[nan]).all() and is_nan_bf16(ref[nan]).all()
    # the closed-form ranges against their own definitions
    assert got[0x0000] == 0x0000 and got[0x8000] == 0x8000       # silu(+-0) = +-0
    assert got[0x7F80] == 0x7F80 and got[0xFF80] == 0x8000       # +inf -> +inf, -inf -> -0
    big = np.arange(0x4300, 0x7F80)                                # 2^7 <= |g| < inf
    assert np.array_equal(got[big], big.astype(np.uint16))
    assert (got[big | 0x8000] == 0x8000).all()
