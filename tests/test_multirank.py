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


def test_bench_launches_replicas_itself():
    """``bench.py --gpus 2`` without a launcher starts two ranks itself
    (torch.distributed.run on 127.0.0.1); with --dry-run they use gloo and
    the CPU oracle, and rank 0 alone prints one line for the whole job"""
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = {k: v for k, v in os.environ.items()
           if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK", "MASTER_ADDR", "MASTER_PORT")}
    out = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--gpus", "2",
                          "--dry-run", "--steps", "2", "--warmup", "3", "--config", "tiny"],
                         capture_output=True, text=True, timeout=600, env=env, cwd=root)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, out.stdout
    rec = json.loads(lines[0])
    assert rec["n_gpus"] == 2
    assert rec["config"]["parallelism"] == "replicas x2"
    assert rec["scaling"] == "weak" and rec["dry_run"] is True
    # value = tokens of both ranks over the slowest rank's time
    assert rec["value"] == pytest.approx(
        rec["config"]["T"] * 2 * rec["steps"] / (rec["ms_per_step"] * rec["steps"] * 1e-3))
