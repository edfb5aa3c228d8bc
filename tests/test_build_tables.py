"""The expert activation's SiLU table is generated on the host at build time
(csrc/gen_silu_table.c); every entry must equal the oracle's correctly
rounded SiLU of the same gate."""

import numpy as np

import oracle
from combine_ep_route_02_b200 import build as B


def test_silu_table_equals_oracle(tmp_path):
    B.generate_tables(str(tmp_path))
    text = (tmp_path / "silu_table.inc").read_text()
    got = np.array([int(v, 16) for v in text.replace("\n", " ").split(",") if v.strip()],
                   dtype=np.uint16)
    assert got.size == 8192
    i = np.arange(8192)
    gate = (((i >> 12) << 15) | (0x3300 + (i & 4095))).astype(np.uint16)
    ref, hard = oracle.silu_bf16_array(gate)
    assert hard.sum() == 0
    assert np.array_equal(got, ref)
