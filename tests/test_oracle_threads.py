"""The oracle's threaded form (token ranges on several host threads, used
for the all-cores CPU baseline) gives the single-thread results bit for
bit: tokens are independent in routing, dispatch and combine."""

import numpy as np
import torch

import oracle
from gen import CONFIGS, Workload


def test_threaded_oracle_equals_single_thread():
    cfg = CONFIGS["skew"].scaled(203)
    wl = Workload(cfg, seed=3)
    args = (wl.logits, wl.bias, cfg.n_group, cfg.topk_group, cfg.topk, cfg.routed_scale,
            cfg.renorm)
    one = oracle.route(*args)
    many = oracle.route(*args, threads=7)
    for a, b in zip(one, many):
        assert np.array_equal(a, b)
    lay = oracle.layout(one[0], cfg.E, cfg.n_phys, cfg.R, wl.phys_of.numpy(), wl.n_rep.numpy())
    d1 = oracle.dispatch(wl.x, lay["slot"], True)
    d7 = oracle.dispatch(wl.x, lay["slot"], True, threads=7)
    assert np.array_equal(d1[0], d7[0]) and np.array_equal(d1[1], d7[1])
    y = torch.randn((cfg.T * cfg.topk, cfg.H), generator=torch.Generator().manual_seed(1))
    y = y.to(torch.bfloat16)
    assert np.array_equal(oracle.combine(y, lay["slot"], one[1]),
                          oracle.combine(y, lay["slot"], one[1], threads=7))
    # more threads than tokens, and no tokens
    small = oracle.route(wl.logits[:3], wl.bias, cfg.n_group, cfg.topk_group, cfg.topk,
                         cfg.routed_scale, cfg.renorm, threads=16)
    assert np.array_equal(small[0], one[0][:3])
    empty = oracle.route(wl.logits[:0], wl.bias, cfg.n_group, cfg.topk_group, cfg.topk,
                         cfg.routed_scale, cfg.renorm, threads=4)
    assert empty[0].shape == (0, cfg.topk)
