"""Helpers shared by the GPU parity tests: run the CUDA path through the C ABI
and the oracle on the same seeded inputs."""

from __future__ import annotations

import numpy as np
import torch

import functools

import oracle
from gen import CONFIGS, Workload

# BF16 combine tolerance: |gpu - oracle| <= ATOL + RTOL * |oracle|
ATOL = 1e-3
RTOL = 1e-2


def u16(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor -> its uint16 bit patterns (host numpy)."""
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def bf16_from_bits(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)


def make_path(cfg, wl: Workload, num_sms: int = 0, row_align: int = 1):
    from combine_ep_route_02_b200 import EpPath
    return EpPath(cfg.T, cfg.H, cfg.E, cfg.n_group, cfg.topk_group, cfg.topk,
                  cfg.routed_scale, cfg.renorm, cfg.R, cfg.fp8,
                  phys_of=wl.phys_of, n_rep=wl.n_rep, num_sms=num_sms, row_align=row_align)


def oracle_route(cfg, wl):
    return oracle.route(wl.logits, wl.bias, cfg.n_group, cfg.topk_group, cfg.topk,
                        cfg.routed_scale, cfg.renorm)


def oracle_layout(cfg, wl, topk_idx, row_align: int = 1):
    po = None if wl.phys_of is None else wl.phys_of.numpy()
    nr = None if wl.n_rep is None else wl.n_rep.numpy()
    return oracle.layout(topk_idx, cfg.E, cfg.n_phys, cfg.R, po, nr, row_align=row_align)


LAYOUT_FIELDS = ("cnt_expert", "expert_off", "rows_rank", "rank_off", "tok_rank",
                 "in_rank", "slot", "src")


def gpu_layout_dict(path):
    return {n: getattr(path, n).cpu().numpy() for n in LAYOUT_FIELDS}


def assert_combine_close(got_bits: np.ndarray, ref_bits: np.ndarray):
    g = bf16_from_bits(got_bits).double().numpy()
    r = bf16_from_bits(ref_bits).double().numpy()
    err = np.abs(g - r)
    bad = err > ATOL + RTOL * np.abs(r)
    assert not bad.any(), (int(bad.sum()), float(err.max()))


@functools.lru_cache(maxsize=8)
def workload(name: str, seed: int = 0) -> Workload:
    """Full-size workloads are reused across tests (inputs are read-only)."""
    return Workload(CONFIGS[name], seed=seed)
