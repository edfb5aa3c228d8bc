#!/usr/bin/env python
"""Throughput of the MoE routing -> layout -> FP8 dispatch -> combine path.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config v3]
                    [--impl ours|reference] [--schedule micro|sequential]

One step = route + dispatch layout + dispatch + combine over one batch of the
named workload (default: DeepSeek-V3 prefill shape, T=8192 tokens, H=7168,
256 experts in 8 groups, top-4 groups, top-8, FP8 1x128 dispatch, BF16
combine).  Inputs are synthetic and seeded; the expert outputs fed to the
combine are a device-resident bf16 N(0,1) buffer standing in for the expert
GEMM, which is not part of this path.

``value`` = tokens of all ranks / (max over ranks of the device time of K
steps).  Multi-GPU runs are independent replicas (one batch per GPU, no data
exchange between GPUs; "scaling": "weak").  ``--impl reference`` times the CPU
oracle on the host cores on a bounded sample of the same workload.
"""

from __future__ import annotations

import argparse
import faulthandler
import json
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from gen import CONFIGS, Workload, device_normal_bf16  # noqa: E402

METRIC = "dispatch+combine tokens/s and achieved HBM GB/s (% of peak) at T=8192,H=7168,top-8"
L2_BYTES = 126 * 1024 * 1024


def algorithmic_bytes(cfg):
    """Bytes each kernel must move per step (no re-reads), by kernel."""
    T, H, k, E, R = cfg.T, cfg.H, cfg.topk, cfg.E, cfg.R
    S = H // 128
    disp = T * 2 * H + T * k * (H + 4 * S if cfg.fp8 else 2 * H) + T * k * 4
    comb = T * k * 2 * H + T * 2 * H + T * k * 8
    route = T * E * 4 + E * 4 + T * k * 8
    layout = T * k * 4 * 3 + T * R + T * k * 4  # ids read twice, slot + src written
    return dict(route=route, layout=layout, dispatch=disp, combine=comb)


def rank_seed(rank: int) -> int:
    """Each replica draws its own batch: the seeded workload with seed = rank."""
    return rank


def reduce_max(x: float, dist, device) -> float:
    """Max of a per-rank float over all ranks (identity without a group)."""
    if dist is None:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def tokens_per_s(T: int, world: int, steps: int, max_ms: float) -> float:
    """Whole-job throughput: the tokens of every rank over the slowest rank's time."""
    return T * world * steps / (max_ms * 1e-3)


def peak_hbm():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


class ClockSampler:
    """Polls SM clock and throttle reasons through NVML (read-only)."""

    def __init__(self, device_index: int, period_s: float = 0.01):
        self.samples = []
        self.ok = False
        self._stop = threading.Event()
        self.window = None
        try:
            import pynvml
            pynvml.nvmlInit()
            props = torch.cuda.get_device_properties(device_index)
            # NVML wants the textual bus id; torch gives its three integers
            bus = "%08X:%02X:%02X.0" % (int(props.pci_domain_id), int(props.pci_bus_id),
                                        int(props.pci_device_id))
            self.h = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
            self.nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # no NVML: report nothing rather than guess
            self.err = str(e)
        self.period = period_s

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                reasons = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                self.samples.append((time.perf_counter(), mhz, reasons))
            except Exception:
                pass
            time.sleep(self.period)

    def start(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()

    def stop(self):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self, t0, t1):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"]}
        inside = [s for s in self.samples if t0 <= s[0] <= t1]
        window = "timed"
        if len(inside) < 3:
            inside = self.samples
            window = "whole run (timed region shorter than the sampling period)"
        names = {
            0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
            0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
            0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
            0x100: "display_clock_setting",
        }
        seen = 0
        for s in inside:
            seen |= s[2]
        reasons = [n for b, n in names.items() if seen & b]
        return {"sm_mhz": statistics.median([s[1] for s in inside]) if inside else None,
                "sm_max_mhz": self.max_mhz, "reasons": reasons, "samples": len(inside),
                "window": window}


def host_cores() -> int:
    """Host cores this process may run on."""
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def cpu_oracle_sample(cfg, wl, y_host_rows, n_tok, threads=1):
    """Oracle route+layout+dispatch+combine on the first n_tok tokens; with
    threads > 1 routing, dispatch and combine run token ranges on that many
    host threads (the layout's counting sweep stays on one)."""
    import oracle
    sub = cfg.scaled(n_tok)
    lg = wl.logits[:n_tok].numpy()
    x = wl.x_rows(0, n_tok)
    t0 = time.perf_counter()
    idx, w, _ = oracle.route(lg, wl.bias, sub.n_group, sub.topk_group, sub.topk,
                             sub.routed_scale, sub.renorm, threads=threads)
    po = None if wl.phys_of is None else wl.phys_of.numpy()
    nr = None if wl.n_rep is None else wl.n_rep.numpy()
    lay = oracle.layout(idx, sub.E, sub.n_phys, sub.R, po, nr)
    oracle.dispatch(x, lay["slot"], sub.fp8, threads=threads)
    oracle.combine(y_host_rows, lay["slot"], w, threads=threads)
    return time.perf_counter() - t0


def free_port() -> int:
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        return sk.getsockname()[1]


def launch_replicas(n: int, argv) -> int:
    """Runs this script as n ranks under torch.distributed.run on this node
    (one process per GPU, rendezvous on 127.0.0.1) and returns their exit
    status.  Used when --gpus N > 1 is given without a launcher."""
    import subprocess
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
           f"--nproc-per-node={n}", "--master-addr", "127.0.0.1",
           f"--master-port={free_port()}", os.path.abspath(__file__), *argv]
    return subprocess.call(cmd)


def run_dry(args, cfg):
    """The multi-rank host logic without a GPU: gloo process group, each rank
    runs the oracle over a small sample of its own batch (seed = rank) as its
    step, the slowest rank's time is the job's, rank 0 prints the line."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    n_tok = min(cfg.T, 32)
    wl = Workload(cfg, seed=rank_seed(rank))
    g = torch.Generator().manual_seed(rank)
    y = torch.randn((n_tok * cfg.topk, cfg.H), generator=g).to(torch.bfloat16)
    for _ in range(args.warmup):
        cpu_oracle_sample(cfg, wl, y, n_tok)
    secs = sum(cpu_oracle_sample(cfg, wl, y, n_tok) for _ in range(args.steps))
    max_ms = reduce_max(secs * 1e3, dist, "cpu")
    if rank == 0:
        value = tokens_per_s(n_tok, world, args.steps, max_ms)
        print(json.dumps({
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": max_ms / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "host oracle (dry run)", "data": "synthetic", "dry_run": True,
            "config": {"workload": cfg.name, "T": n_tok, "H": cfg.H, "E": cfg.E,
                       "topk": cfg.topk, "parallelism": f"replicas x{world}",
                       "note": "no GPU: each rank's step is the CPU oracle on its own batch"}}),
            flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


def run_reference(args, cfg):
    """The oracle on the host cores: each step is a bounded token sample."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    n_tok = min(cfg.T, args.ref_tokens)
    wl = Workload(cfg)
    g = torch.Generator().manual_seed(7)
    y = torch.randn((n_tok * cfg.topk, cfg.H), generator=g).to(torch.bfloat16)
    cores = host_cores()
    for _ in range(args.warmup):
        cpu_oracle_sample(cfg, wl, y, n_tok, threads=cores)
    times = [cpu_oracle_sample(cfg, wl, y, n_tok, threads=cores) for _ in range(args.steps)]
    tot = sum(times)
    value = n_tok * args.steps / tot
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * tot / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "fp8-e4m3 dispatch / bf16 combine, fp32 accumulate",
        "data": "synthetic",
        "config": {"workload": cfg.name, "T": cfg.T, "H": cfg.H, "E": cfg.E, "topk": cfg.topk,
                   "sample_tokens": n_tok},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": f"first {n_tok} of {cfg.T} tokens per step, routing, "
                                   f"dispatch and combine split over {cores} host threads"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default="v3", choices=sorted(CONFIGS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--schedule", default="micro", choices=["micro", "sequential"],
                    help="micro: micro-batches in flight over three buffer sets (route+layout "
                         "of later batches overlap dispatch+combine of batch i); sequential: "
                         "one step after the other on one stream")
    ap.add_argument("--num-sms", type=int, default=0)
    ap.add_argument("--split-sms", default="",
                    help="micro-batch schedule: 'd,c' runs dispatch of batch i+1 on d SMs next "
                         "to combine of batch i on c SMs; empty = one after the other")
    ap.add_argument("--ref-tokens", type=int, default=512,
                    help="tokens per oracle step (--impl reference and cpu_baseline)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--tokens", type=int, default=0,
                    help="run the workload with this many tokens instead (small cases for "
                         "profiler captures); 0 = the workload's own T")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-backward", action="store_true",
                    help="skip timing the training backward (dispatch/combine backward)")
    ap.add_argument("--no-gemm-layout", action="store_true",
                    help="skip timing the GEMM layout (padded rows) and the expert activation")
    ap.add_argument("--row-align", type=int, default=128,
                    help="row tile of the GEMM layout timed after the step")
    ap.add_argument("--peer-ranks", type=int, default=8,
                    help="also time the peer-memory expert-parallel dispatch and combine with "
                         "this many ranks on this GPU (0 = skip)")
    ap.add_argument("--dry-run", action="store_true",
                    help="no GPU: check the multi-rank launch, the max-over-ranks timing and "
                         "the output line with gloo ranks running the CPU oracle")
    args = ap.parse_args()
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        sys.exit(launch_replicas(args.gpus, sys.argv[1:]))
    faulthandler.enable()
    cfg = CONFIGS[args.config]
    if args.tokens > 0:
        cfg = cfg.scaled(args.tokens)
    if args.warmup < 3:
        print("warning: fewer than 3 warm-up steps", file=sys.stderr)

    if args.impl == "reference":
        run_reference(args, cfg)
        return
    if args.dry_run:
        run_dry(args, cfg)
        return

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))

    from combine_ep_route_02_b200 import EpPath

    wl = Workload(cfg, seed=rank_seed(rank))
    x_h = wl.x.pin_memory()
    lg_h = wl.logits.pin_memory()
    b_h = wl.bias.pin_memory()
    x, lg, bias = x_h.cuda(), lg_h.cuda(), b_h.cuda()
    y = device_normal_bf16(cfg.T * cfg.topk, cfg.H, seed=rank_seed(rank))
    path = EpPath(cfg.T, cfg.H, cfg.E, cfg.n_group, cfg.topk_group, cfg.topk, cfg.routed_scale,
                  cfg.renorm, cfg.R, cfg.fp8, phys_of=wl.phys_of, n_rep=wl.n_rep,
                  num_sms=args.num_sms)
    stream = torch.cuda.current_stream()
    ab = algorithmic_bytes(cfg)
    step_bytes = sum(ab.values())
    flush = step_bytes < 2 * L2_BYTES
    # L2 flush between steps: write 256 MiB, then read another 256 MiB, so
    # that L2 holds none of the step's data and no dirty lines whose write-back
    # the next step would pay for
    flush_w = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device="cuda") if flush else None
    flush_r = torch.ones(64 * 1024 * 1024, dtype=torch.float32, device="cuda") if flush else None

    def flush_l2(i):
        flush_w.fill_(i & 0xFF)
        flush_r.sum()

    def barrier():
        if dist is not None:
            dist.barrier()

    def step():
        path.step(x, lg, bias, y)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    path.check_status()

    K = args.steps

    def events(n=None):
        return [torch.cuda.Event(enable_timing=True) for _ in range(K if n is None else n)]

    def total_ms(a, b):
        return reduce_max(sum(x.elapsed_time(y) for x, y in zip(a, b)), dist, "cuda")

    s0, s1, d0, d1, c0, c1 = events(), events(), events(), events(), events(), events()
    sampler = ClockSampler(local)
    sampler.start()
    barrier()
    torch.cuda.synchronize()
    t_wall0 = time.perf_counter()

    # 1. eager launches on one stream, events around route+layout, dispatch
    #    and combine (the per-kernel attribution and the roofline); a batch
    #    small enough for the one-kernel route+layout+dispatch runs that
    #    kernel between s0 and d1 (d0 is recorded just before it)
    fused = path.fused_route_dispatch()
    for i in range(K):
        if flush:
            flush_l2(i)  # evict the previous step's data from L2
        s0[i].record(stream)
        if fused:
            d0[i].record(stream)
            path.route_dispatch(lg, bias, x)
        else:
            path.route_layout(lg, bias)
            d0[i].record(stream)
            path.dispatch(x)
        d1[i].record(stream)
        c0[i].record(stream)
        path.combine(y)
        c1[i].record(stream)
        s1[i].record(stream)
    torch.cuda.synchronize()
    barrier()
    path.check_status()
    eager_ms = total_ms(s0, s1)

    # 2. the same step captured once as a CUDA graph and replayed: no host
    #    launch cost per kernel (what bounds small batches when eager)
    gs = torch.cuda.Stream()
    gs.wait_stream(stream)
    with torch.cuda.stream(gs):
        step()
    stream.wait_stream(gs)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    for _ in range(args.warmup):
        graph.replay()
    g0, g1 = events(), events()
    torch.cuda.synchronize()
    barrier()
    for i in range(K):
        if flush:
            flush_l2(i)
        g0[i].record(stream)
        graph.replay()
        g1[i].record(stream)
    torch.cuda.synchronize()
    barrier()
    path.check_status()
    graph_ms = total_ms(g0, g1)
    seq_ms = graph_ms
    value_seq = tokens_per_s(cfg.T, world, K, seq_ms)

    # 3. the same K batches with micro-batches in flight (three buffer sets)
    micro_ms = None
    # the two-stream schedule has no L2 flush between steps, so it is only
    # timed when a step's data is larger than L2 anyway
    if args.schedule == "micro" and not flush:
        from combine_ep_route_02_b200 import EpMicroBatchPipeline
        from combine_ep_route_02_b200.path import EpPath as _EpPath

        def make_path():
            return _EpPath(cfg.T, cfg.H, cfg.E, cfg.n_group, cfg.topk_group, cfg.topk,
                           cfg.routed_scale, cfg.renorm, cfg.R, cfg.fp8, phys_of=wl.phys_of,
                           n_rep=wl.n_rep, num_sms=args.num_sms)
        split = None
        if args.split_sms:
            d_sms, c_sms = (int(v) for v in args.split_sms.split(","))
            split = (d_sms, c_sms)
        mb = EpMicroBatchPipeline(make_path, split_sms=split)
        mb.run([x] * args.warmup, [lg] * args.warmup, [bias] * args.warmup, [y] * args.warmup)
        torch.cuda.synchronize()
        barrier()
        m0 = torch.cuda.Event(enable_timing=True)
        m1 = torch.cuda.Event(enable_timing=True)
        m0.record(mb.s_route)
        mb.run([x] * K, [lg] * K, [bias] * K, [y] * K)
        m1.record(mb.s_last)
        torch.cuda.synchronize()
        barrier()
        mb.check_status()
        micro_ms = reduce_max(m0.elapsed_time(m1), dist, "cuda")
        del mb
    # backward pass of the training step (dispatch-backward = combine of the
    # gradient rows, combine-backward = scaled scatter + weight gradients),
    # events around each call on the launching stream
    backward = None
    if not args.no_backward:
        from combine_ep_route_02_b200 import ep_combine_backward, ep_dispatch_backward
        g_out = device_normal_bf16(cfg.T, cfg.H, seed=100 + rank)
        g_x = torch.empty((cfg.T, cfg.H), dtype=torch.bfloat16, device="cuda")
        g_y = torch.empty((cfg.T * cfg.topk, cfg.H), dtype=torch.bfloat16, device="cuda")
        g_w = torch.empty((cfg.T, cfg.topk), dtype=torch.float32, device="cuda")
        Kb = max(3, min(K, 50))
        b0, b1, b2 = (events(Kb) for _ in range(3))
        for i in range(args.warmup + Kb):
            j = i - args.warmup
            if flush:
                flush_l2(i)
            if j >= 0:
                b0[j].record(stream)
            ep_dispatch_backward(y, path.slot, cfg.T, cfg.H, cfg.topk, g_x,
                                 dev_status=path.copy_status)
            if j >= 0:
                b1[j].record(stream)
            ep_combine_backward(g_out, y, path.slot, path.topk_w, cfg.T, cfg.H, cfg.topk, g_y, g_w,
                                dev_status=path.copy_status)
            if j >= 0:
                b2[j].record(stream)
        torch.cuda.synchronize()
        path.check_status()
        db_ms = statistics.mean(a.elapsed_time(b) for a, b in zip(b0, b1))
        cb_ms = statistics.mean(a.elapsed_time(b) for a, b in zip(b1, b2))
        T_, H_, k_ = cfg.T, cfg.H, cfg.topk
        db_bytes = T_ * k_ * 2 * H_ + T_ * 2 * H_ + T_ * k_ * 4
        cb_bytes = T_ * 2 * H_ + 2 * T_ * k_ * 2 * H_ + T_ * k_ * 12
        backward = {"dispatch_backward_us": db_ms * 1e3,
                    "dispatch_backward_gbs": db_bytes / (db_ms * 1e-3) / 1e9,
                    "combine_backward_us": cb_ms * 1e3,
                    "combine_backward_gbs": cb_bytes / (cb_ms * 1e-3) / 1e9,
                    "tokens_per_s": T_ * world / ((db_ms + cb_ms) * 1e-3)}
        del g_out, g_x, g_y, g_w
    # GEMM layout: expert rows padded to the grouped GEMM's row tile, and the
    # expert activation silu(gate) * up -> e4m3 + 1x128 scales between the two
    # expert GEMMs, over the rows the device-side counts select
    gemm = None
    if not args.no_gemm_layout:
        A, I = args.row_align, cfg.inter
        pa = EpPath(cfg.T, cfg.H, cfg.E, cfg.n_group, cfg.topk_group, cfg.topk,
                    cfg.routed_scale, cfg.renorm, cfg.R, cfg.fp8, phys_of=wl.phys_of,
                    n_rep=wl.n_rep, num_sms=args.num_sms, row_align=A)
        gate_up = device_normal_bf16(pa.n_recv, 2 * I, seed=200 + rank)
        act = torch.empty((pa.n_recv, I), dtype=torch.float8_e4m3fn, device="cuda")
        act_sc = torch.empty((pa.n_recv, I // 128), dtype=torch.float32, device="cuda")
        V = cfg.T * cfg.topk
        act_bytes = V * (4 * I + I + 4 * (I // 128)) + pa.P * 8
        act_flush = act_bytes < 2 * L2_BYTES
        if act_flush and flush_w is None:
            flush_w = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device="cuda")
            flush_r = torch.ones(64 * 1024 * 1024, dtype=torch.float32, device="cuda")
        Ka = max(3, min(K, 50))
        a0, a1, a2 = (events(Ka) for _ in range(3))
        for i in range(args.warmup + Ka):
            j = i - args.warmup
            if act_flush:
                flush_l2(i)
            if j >= 0:
                a0[j].record(stream)
            pa.route_layout(lg, bias)
            if j >= 0:
                a1[j].record(stream)
            pa.activation(gate_up, act, act_sc)
            if j >= 0:
                a2[j].record(stream)
        torch.cuda.synchronize()
        pa.check_status()
        rl_a_ms = statistics.mean(a.elapsed_time(b) for a, b in zip(a0, a1))
        act_ms = statistics.mean(a.elapsed_time(b) for a, b in zip(a1, a2))
        used = int(pa.expert_off[-1].item())
        act_gbs = act_bytes / (act_ms * 1e-3) / 1e9
        pk, pk_kind = peak_hbm()
        gemm = {"row_align": A, "I": I, "recv_rows_capacity": pa.n_recv,
                "recv_rows_used": used, "padding_rows": used - V,
                "route_layout_us": rl_a_ms * 1e3,
                "silu_mul_us": act_ms * 1e3, "silu_mul_gbs": act_gbs,
                "silu_mul_frac": act_gbs / pk,
                "silu_mul_bytes": act_bytes,
                "l2": "flushed before each call" if act_flush else "inputs larger than L2"}
        del pa, gate_up, act, act_sc
    t_wall1 = time.perf_counter()
    sampler.stop()
    tot_ms = micro_ms if micro_ms is not None else seq_ms
    value = tokens_per_s(cfg.T, world, K, tot_ms)

    peak, peak_kind = peak_hbm()
    roofline = None
    extra = {}
    if True:
        comb_ms = statistics.mean(a.elapsed_time(b) for a, b in zip(c0, c1))
        disp_ms = statistics.mean(a.elapsed_time(b) for a, b in zip(d0, d1))
        rl_ms = statistics.mean(a.elapsed_time(b) for a, b in zip(s0, d0))
        comb_gbs = ab["combine"] / (comb_ms * 1e-3) / 1e9
        # the fused kernel moves the routing, layout and dispatch bytes
        disp_bytes = ab["dispatch"] + (ab["route"] + ab["layout"] if fused else 0)
        disp_gbs = disp_bytes / (disp_ms * 1e-3) / 1e9
        peak_src = (f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs copy)" if peak_kind == "measured"
                    else "fallback 6650 GB/s")
        # the dominant kernel of the step by event time
        if comb_ms >= disp_ms:
            dom, dom_gbs, dom_bytes, dom_ms = "combine_kernel", comb_gbs, ab["combine"], comb_ms
        else:
            dom = ("route_dispatch_small_kernel" if fused else "dispatch_fp8_tma_kernel"
                   if cfg.fp8 else "dispatch_bf16_kernel")
            dom_gbs, dom_bytes, dom_ms = disp_gbs, disp_bytes, disp_ms
        roofline = {"bound": "hbm", "kernel": dom, "achieved": dom_gbs,
                    "peak": peak, "unit": "GB/s", "frac": dom_gbs / peak,
                    "peak_source": peak_src,
                    "algorithmic_bytes_per_launch": dom_bytes,
                    "launch_us": dom_ms * 1e3,
                    "timing": "CUDA events on the launching stream around each launch, "
                              "mean over the K eager steps",
                    # DRAM bytes need a profiler's counters, which this run does
                    # not collect
                    "traffic": None,
                    "traffic_source": ("ncu capture of this kernel, one launch, in profiles/ "
                                       "(" + ("route_dispatch_small_kernel_v3_decode.md"
                                              if dom == "route_dispatch_small_kernel" else
                                              "combine_kernel_v3_T2048.md"
                                              if dom == "combine_kernel" else
                                              "dispatch_fp8_tma_kernel_v3_T2048.md") + ")")}
        dc_ms = comb_ms + disp_ms
        extra = {
            "route_layout_us": None if fused else rl_ms * 1e3,
            "dispatch_us": None if fused else disp_ms * 1e3,
            "route_dispatch_us": disp_ms * 1e3 if fused else None,
            "combine_us": comb_ms * 1e3,
            "dispatch_gbs": disp_gbs, "combine_gbs": comb_gbs,
            "dispatch_combine_tokens_per_s": cfg.T * world / (dc_ms * 1e-3),
            "dispatch_combine_gbs": (ab["dispatch"] + ab["combine"]) / (dc_ms * 1e-3) / 1e9,
            "dispatch_combine_frac_of_peak": (ab["dispatch"] + ab["combine"]) / (dc_ms * 1e-3)
            / 1e9 / peak,
            "step_gbs": step_bytes / (tot_ms / K * 1e-3) / 1e9,
            "step_us": tot_ms / K * 1e3,
        }

    # expert parallelism over peer memory, every rank on this GPU: the
    # workload's tokens split over `peer_ranks` ranks (R = that many), each
    # with its own buffers addressed through the rank tables a multi-GPU
    # group uses; events around the fused quantise + store dispatch and the
    # gathering combine (stores and loads stay in this GPU's HBM here, where
    # a multi-GPU group crosses NVLink)
    peer = None
    if args.peer_ranks > 1 and cfg.fp8 and cfg.T % args.peer_ranks == 0 and world == 1:
        import dataclasses

        from combine_ep_route_02_b200 import EpPeerRanks
        Wp = args.peer_ranks
        pcfg = dataclasses.replace(cfg.scaled(cfg.T // Wp), R=Wp)
        pwls = [Workload(pcfg, seed=1000 + r) for r in range(Wp)]
        ppaths = [EpPath(pcfg.T, pcfg.H, pcfg.E, pcfg.n_group, pcfg.topk_group, pcfg.topk,
                         pcfg.routed_scale, pcfg.renorm, Wp, True, phys_of=w.phys_of,
                         n_rep=w.n_rep) for w in pwls]
        for pp_, w in zip(ppaths, pwls):
            pp_.route_layout(w.logits.cuda(), w.bias.cuda())
        grp = EpPeerRanks.local(ppaths, pcfg.H)
        pxs = [w.x.cuda() for w in pwls]
        pouts = [torch.empty((pcfg.T, pcfg.H), dtype=torch.bfloat16, device="cuda")
                 for _ in range(Wp)]
        grp.set_inputs(pxs, pouts)
        for i, yq in enumerate(grp.y):
            yq.copy_(device_normal_bf16(grp.cap, pcfg.H, seed=2000 + i))
        Kp = max(3, min(K, 50))
        qc, q0, q1, q2, q3 = (events(Kp) for _ in range(5))
        for i in range(args.warmup + Kp):
            j = i - args.warmup
            if j >= 0:
                qc[j].record(stream)
            grp.counts()
            if j >= 0:
                q0[j].record(stream)
            grp.dispatch()
            if j >= 0:
                q1[j].record(stream)
            grp.wait_dispatch()
            grp.experts_ready()
            if j >= 0:
                q2[j].record(stream)
            grp.combine()
            if j >= 0:
                q3[j].record(stream)
        torch.cuda.synchronize()
        if any(grp.check_status()):
            raise RuntimeError(f"peer step status {grp.check_status()}")
        pn_ms = statistics.mean(a.elapsed_time(b) for a, b in zip(qc, q0))
        pd_ms = statistics.mean(a.elapsed_time(b) for a, b in zip(q0, q1))
        pc_ms = statistics.mean(a.elapsed_time(b) for a, b in zip(q2, q3))
        pab = algorithmic_bytes(pcfg)
        pd_bytes, pc_bytes = pab["dispatch"] * Wp, pab["combine"] * Wp
        peer = {"ranks": Wp, "tokens_per_rank": pcfg.T, "counts_us": pn_ms * 1e3,
                "dispatch_us": pd_ms * 1e3, "dispatch_gbs": pd_bytes / (pd_ms * 1e-3) / 1e9,
                "combine_us": pc_ms * 1e3, "combine_gbs": pc_bytes / (pc_ms * 1e-3) / 1e9,
                "dispatch_combine_tokens_per_s": cfg.T / ((pd_ms + pc_ms) * 1e-3),
                "note": "all ranks on one GPU (one launch covers them); algorithmic bytes "
                        "as for dispatch and combine, summed over the ranks"}
        del grp, ppaths, pxs, pouts

    # end to end through the public API: every step uploads its inputs from
    # pinned host memory and downloads its result; EpHostPipeline overlaps
    # those copies with the neighbouring steps' compute
    e2e = None
    if not args.no_e2e:
        from combine_ep_route_02_b200 import EpHostPipeline
        pipe = EpHostPipeline(path)
        Ke = max(4, min(K, 50))
        outs = [torch.empty((cfg.T, cfg.H), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
        xs, lgs, bs = [x_h] * Ke, [lg_h] * Ke, [b_h] * Ke
        ohs = [outs[i & 1] for i in range(Ke)]
        pipe.run(xs[:4], lgs[:4], bs[:4], ohs[:4], y)  # warm-up
        torch.cuda.synchronize()
        barrier()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(pipe.s_h2d)
        pipe.run(xs, lgs, bs, ohs, y)
        e1.record(pipe.s_d2h)
        torch.cuda.synchronize()
        barrier()
        ems = reduce_max(e0.elapsed_time(e1), dist, "cuda")
        h2d = x_h.numel() * 2 + lg_h.numel() * 4 + b_h.numel() * 4
        e2e = {"value": tokens_per_s(cfg.T, world, Ke, ems), "unit": "tokens/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": outs[0].numel() * 2,
               "steps": Ke, "overlap": "H2D(i+1) and D2H(i-1) overlap compute(i)"}
        path.check_status()

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        # whole passes of the oracle over the workload's batch, on one thread
        # and then on every host core, until about 10 s of CPU work each (at
        # most 8 passes)
        yh = y.cpu()
        cores = host_cores()

        def oracle_rate(threads):
            secs, passes = 0.0, 0
            while passes < 8 and (secs < 10.0 or passes == 0):
                secs += cpu_oracle_sample(cfg, wl, yh, cfg.T, threads=threads)
                passes += 1
            return cfg.T * passes / secs, passes, secs

        v1, p1, s1_ = oracle_rate(1)
        vn, pn, sn = oracle_rate(cores)
        cpu = {"value": vn, "unit": "tokens/s", "cores": cores, "kind": "oracle",
               "sample": f"{pn} pass(es) of route+layout+dispatch+combine over all {cfg.T} "
                         f"tokens of the same batch, routing, dispatch and combine split "
                         f"over {cores} host threads ({sn:.1f} s)",
               "single_thread": {"value": v1, "cores": 1,
                                 "sample": f"{p1} pass(es) over all {cfg.T} tokens, one "
                                           f"thread ({s1_:.1f} s)"}}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": tot_ms / K, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None,
            "dtype": "fp8-e4m3 dispatch / bf16 combine, fp32 accumulate",
            "data": "synthetic (seeded SplitMix64 / Box-Muller inputs; expert outputs bf16 N(0,1))",
            "config": {"workload": cfg.name, "T": cfg.T, "H": cfg.H, "E": cfg.E,
                       "P": cfg.n_phys, "R": cfg.R, "n_group": cfg.n_group,
                       "topk_group": cfg.topk_group, "topk": cfg.topk, "fp8": cfg.fp8,
                       "routed_scale": cfg.routed_scale, "cuda_graph": micro_ms is None,
                       "l2": ("flushed before each step (256 MiB written, then another "
                              "256 MiB read, outside the step's events)"
                              if flush else
                              f"inputs larger than L2 ({step_bytes / 1e9:.2f} GB moved per step)"),
                       "parallelism": f"replicas x{world}",
                       "schedule": ("micro-batches in flight over three buffer sets: "
                                    "route+layout of later batches on one stream overlap "
                                    "dispatch+combine of batch i on another"
                                    if micro_ms is not None else
                                    "sequential, one stream, step replayed as a CUDA graph")},
            "value_sequential": value_seq, "ms_per_step_sequential": seq_ms / K,
            "value_sequential_eager": tokens_per_s(cfg.T, world, K, eager_ms),
            "ms_per_step_sequential_eager": eager_ms / K,
            "gpu_launches": path.kernels_per_step() * K,
            "gpu_launches_note": "per timed pass of K steps (each of the eager, graph and "
                                 "micro-batch passes launches this many)",
            "roofline": roofline,
            "e2e": e2e,
            "cpu_baseline": cpu,
            "backward": backward,
            "gemm_layout": gemm,
            "peer_ep": peer,
            "clocks": sampler.summary(t_wall0, t_wall1),
            "wall_s_timed": t_wall1 - t_wall0,
            **extra,
        }
        print(json.dumps(line), flush=True)
    del graph
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
