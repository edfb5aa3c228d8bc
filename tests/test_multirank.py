"""The multi-GPU path is replicas only: every rank runs the whole path on its
own batch (seed = rank) and the job's time is the slowest rank's.  These
world-size-2 gloo runs check that host logic on CPU: the ranks' batches
differ, each rank's oracle result is reproducible from its seed alone, and
the max-over-ranks reduction and throughput aggregation agree with a direct
computation."""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import sys
        sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
        import bench
        import oracle
        from gen import CONFIGS, Workload
        cfg = CONFIGS["ds16b"].scaled(64)
        wl = Workload(cfg, seed=bench.rank_seed(rank))
        idx, w, _ = oracle.route(wl.logits, wl.bias, cfg.n_group, cfg.topk_group, cfg.topk,
                                 cfg.routed_scale, cfg.renorm)
        lay = oracle.layout(idx, cfg.E, cfg.E, cfg.R)
        rx, rs = oracle.dispatch(wl.x, lay["slot"], True)
        digest = float(np.float64(rx.sum()) + np.float64(rs.astype(np.float64).sum()))
        fake_ms = 10.0 + 7.0 * rank          # stands in for this rank's device time
        mx = bench.reduce_max(fake_ms, dist, "cpu")
        gathered = [torch.zeros(2, dtype=torch.float64) for _ in range(world)]
        dist.all_gather(gathered, torch.tensor([digest, fake_ms], dtype=torch.float64))
        value = bench.tokens_per_s(cfg.T, world, 5, mx)
        np.save(os.path.join(out_dir, f"rank{rank}.npy"),
                np.array([digest, mx, value] + [g[0].item() for g in gathered] +
                         [g[1].item() for g in gathered]))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2])
def test_replicas_gloo(tmp_path, world):
    port = _free_port()
    mp.start_processes(_rank_main, args=(world, port, str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    res = [np.load(tmp_path / f"rank{r}.npy") for r in range(world)]
    digests = [r[0] for r in res]
    assert len(set(digests)) == world           # every rank dispatched its own batch
    for r in res:
        assert r[1] == 10.0 + 7.0 * (world - 1)  # max over ranks
        assert r[2] == pytest.approx(64 * world * 5 / (r[1] * 1e-3))
        assert list(r[3:3 + world]) == digests  # every rank saw the same digests
    # a rank's result depends on its seed only: recompute rank 1 here
    import bench
    import oracle
    from gen import CONFIGS, Workload
    cfg = CONFIGS["ds16b"].scaled(64)
    wl = Workload(cfg, seed=bench.rank_seed(1))
    idx, w, _ = oracle.route(wl.logits, wl.bias, cfg.n_group, cfg.topk_group, cfg.topk,
                             cfg.routed_scale, cfg.renorm)
    lay = oracle.layout(idx, cfg.E, cfg.E, cfg.R)
    rx, rs = oracle.dispatch(wl.x, lay["slot"], True)
    assert float(np.float64(rx.sum()) + np.float64(rs.astype(np.float64).sum())) == digests[1]
