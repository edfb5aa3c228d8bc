"""The allocation-free layout entry point gives the same results as the
ordinary one.

ep_dispatch_layout_noalloc serves callers that cannot allocate device memory
at the call site (an engine plugin's enqueue hook, a framework operator with
no access to its caching allocator, a decode step that cannot pay for the
device synchronisation cudaMalloc may cause).  It keeps its scratch in a
fixed device array inside the library instead of a caller workspace.  This
file is collected last so that a failure here cannot hide another test.
"""

import numpy as np
import pytest
import torch

from combine_ep_route_02_b200 import _binding as B

pytestmark = pytest.mark.gpu

FIELDS = ("cnt_expert", "expert_off", "rows_rank", "rank_off", "tok_rank", "in_rank", "slot",
          "src", "dev_status")


def _outputs(T, k, P, R):
    i32 = dict(dtype=torch.int32, device="cuda")
    # filled with garbage so that an output the call forgets to write shows up
    return dict(cnt_expert=torch.full((P,), -9, **i32),
                expert_off=torch.full((P + 1,), -9, **i32),
                rows_rank=torch.full((R,), -9, **i32), rank_off=torch.full((R + 1,), -9, **i32),
                tok_rank=torch.full((R,), -9, **i32),
                in_rank=torch.full((T, R), 7, dtype=torch.uint8, device="cuda"),
                slot=torch.full((T, k), -9, **i32), src=torch.full((T * k,), -9, **i32),
                dev_status=torch.full((1,), -9, **i32))


def _ids(T, k, E, seed, bad=False):
    rng = np.random.default_rng(seed)
    idx = np.argsort(rng.random((T, E)), axis=1)[:, :k].astype(np.int32)
    if bad:
        idx[T // 2, 0] = E + 3  # reported through dev_status, slot -1
    return torch.from_numpy(idx).cuda()


def _with_workspace(idx, T, k, E, P, R, phys_of, n_rep, max_rep):
    o = _outputs(T, k, P, R)
    ws = torch.empty(B.ep_workspace_size(T, k, P, R), dtype=torch.uint8, device="cuda")
    B.ep_dispatch_layout(idx, T, k, E, P, R, phys_of, n_rep, max_rep, o["cnt_expert"],
                         o["expert_off"], o["rows_rank"], o["rank_off"], o["tok_rank"],
                         o["in_rank"], o["slot"], o["src"], ws, o["dev_status"])
    return o


def _without(idx, T, k, E, P, R, phys_of, n_rep, max_rep):
    o = _outputs(T, k, P, R)
    B.ep_dispatch_layout_noalloc(idx, T, k, E, P, R, phys_of, n_rep, max_rep, o["cnt_expert"],
                                 o["expert_off"], o["rows_rank"], o["rank_off"], o["tok_rank"],
                                 o["in_rank"], o["slot"], o["src"], o["dev_status"])
    return o


def test_noalloc_layout_matches_workspace_layout_twice():
    assert torch.cuda.is_available()
    # two calls in a row with different shapes: the second finds the first
    # call's data in the shared scratch and must not depend on it
    cases = [
        dict(T=16384, k=8, E=256, P=288, R=32, seed=1, replicas=True, bad=False),
        dict(T=1000, k=6, E=64, P=64, R=8, seed=2, replicas=False, bad=True),
        # more than 64 tiles: the column-scan kernel rewrites the per-tile
        # histograms in place, over what the previous call left there
        dict(T=40000, k=8, E=256, P=256, R=8, seed=3, replicas=False, bad=False),
    ]
    for c in cases:
        T, k, E, P, R = c["T"], c["k"], c["E"], c["P"], c["R"]
        idx = _ids(T, k, E, c["seed"], c["bad"])
        if c["replicas"]:
            from gen import CONFIGS, Workload
            wl = Workload(CONFIGS["skew"].scaled(8))
            phys_of, n_rep, max_rep = wl.phys_of.cuda(), wl.n_rep.cuda(), 2
        else:
            phys_of = n_rep = None
            max_rep = 0
        ref = _with_workspace(idx, T, k, E, P, R, phys_of, n_rep, max_rep)
        got = _without(idx, T, k, E, P, R, phys_of, n_rep, max_rep)
        torch.cuda.synchronize()
        for n in FIELDS:
            assert torch.equal(got[n], ref[n]), n
        assert int(got["dev_status"].item()) == (B.EP_DEV_BAD_EXPERT if c["bad"] else 0)


def test_noalloc_rejects_sizes_beyond_its_scratch():
    P, R, k = 256, 8, 8
    T = 3000000  # needs more than the 4 MiB of fixed scratch
    assert B.ep_workspace_size(T, k, P, R) > 4 << 20
    st = B.lib().ep_dispatch_layout_noalloc(None, T, k, P, P, R, None, None, 0, *([None] * 8),
                                            None, None)
    assert st == B.EP_ERR_UNSUPPORTED
