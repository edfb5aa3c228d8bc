"""Expert parallelism across processes (two gloo ranks on CPU): each rank
lays out its own batch for R = 2 owner ranks, the dispatch exchange delivers
to each rank exactly the rows of every source that its experts own (with the
per-source, per-expert counts), and the combine exchange returns the expert
outputs to their sources in receive-row order.  The rows are produced by the
oracle here because the test has no GPU; the exchange only moves bytes."""

import dataclasses
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_batch(rank, align, world=2):
    """this rank's layout and FP8 receive rows (recomputable from the seed)"""
    import oracle
    from gen import CONFIGS, Workload
    E = 64 if world == 2 else 48
    cfg = dataclasses.replace(CONFIGS["ds16b"].scaled(96), R=world, E=E)
    wl = Workload(cfg, seed=1000 + rank)
    idx, w, _ = oracle.route(wl.logits, wl.bias, cfg.n_group, cfg.topk_group, cfg.topk,
                             cfg.routed_scale, cfg.renorm)
    lay = oracle.layout(idx, cfg.E, cfg.E, cfg.R, row_align=align)
    n_rows = cfg.T * cfg.topk + cfg.E * (align - 1)
    rx, rs = oracle.dispatch(wl.x, lay["slot"], True, n_rows=n_rows)
    return cfg, lay, rx, rs, w


def _expert(rx_rows, rs_rows):
    """a stand-in expert: bf16 of the dequantised row (exact in fp32)"""
    import oracle
    codes = rx_rows.astype(np.uint8)
    dec = np.vectorize(oracle.e4m3_decode, otypes=[np.float32])(codes)
    h = codes.shape[1]
    vals = dec * np.repeat(rs_rows, 128, axis=1)[:, :h]
    return oracle.bf16_encode_array(vals.astype(np.float32))


def _rank_main(rank, world, port, align, out_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import sys
        sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
        from combine_ep_route_02_b200.exchange import (combine_exchange, dispatch_exchange,
                                                       exchange_plan)
        cfg, lay, rx, rs, _ = _rank_batch(rank, align, world)
        plan = exchange_plan(lay["rows_rank"], lay["cnt_expert"])
        got_x = dispatch_exchange(torch.from_numpy(rx), plan)
        got_s = dispatch_exchange(torch.from_numpy(rs), plan)
        # the experts of this rank process what they received
        y_local = _expert(got_x.numpy(), got_s.numpy())
        y_back = combine_exchange(torch.from_numpy(y_local.view(np.int16)).view(torch.bfloat16),
                                  plan)
        np.savez(os.path.join(out_dir, f"rank{rank}.npz"), got_x=got_x.numpy(),
                 got_s=got_s.numpy(), recv_cnt=plan.recv_cnt.numpy(),
                 recv_splits=np.array(plan.recv_splits),
                 y_back=y_back.view(torch.int16).numpy().view(np.uint16))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def _check(tmp_path, align, world=2):
    port = _free_port()
    mp.start_processes(_rank_main, args=(world, port, align, str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    batches = [_rank_batch(r, align, world) for r in range(world)]
    for me in range(world):
        res = np.load(tmp_path / f"rank{me}.npz")
        parts_x, parts_s, cnts = [], [], []
        for src in range(world):
            cfg, lay, rx, rs, _ = batches[src]
            a, b = lay["rank_off"][me], lay["rank_off"][me + 1]
            parts_x.append(rx[a:b])
            parts_s.append(rs[a:b])
            epr = cfg.E // world
            cnts.append(lay["cnt_expert"][me * epr:(me + 1) * epr])
        assert np.array_equal(res["got_x"], np.concatenate(parts_x))
        assert np.array_equal(res["got_s"], np.concatenate(parts_s))
        assert np.array_equal(res["recv_cnt"], np.stack(cnts))
        assert list(res["recv_splits"]) == [len(p) for p in parts_x]
        # the outputs came back to their source in receive-row order
        cfg, lay, rx, rs, _ = batches[me]
        n = int(lay["rank_off"][-1])
        assert np.array_equal(res["y_back"], _expert(rx[:n], rs[:n]))


def test_exchange_two_ranks(tmp_path):
    _check(tmp_path, 1)


def test_exchange_two_ranks_gemm_layout(tmp_path):
    _check(tmp_path, 16)


def test_exchange_three_ranks(tmp_path):
    _check(tmp_path, 8, world=3)
