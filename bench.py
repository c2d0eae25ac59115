#!/usr/bin/env python3
"""Benchmark of the fused K-quant dequant-GEMV path (libkq) on B200.

Default workload: the Llama-3.1-8B-shaped decode chain at batch 1 -- per
layer Wq|Wk|Wv (6144 x 4096), Wo (4096 x 4096), Wgate|Wup (28672 x 4096) in
Q4_K and Wdown (4096 x 14336) in Q6_K, 32 layers, 4.41 GB of weights, which
is larger than L2, so every step streams the weights from HBM.  One step is
one pass of the whole chain (128 fused GEMV launches, replayed as one CUDA
graph).  Metric: weight GB/s (algorithmic weight bytes / time) and
layer-chain tokens/s.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
  python bench.py --impl reference ...   # the CPU oracle on a bounded sample

Multi-GPU: the chain does not shard in this benchmark; N ranks run N
independent replicas (weak scaling) with no collective on the data path.
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "K-quant dequant-GEMV weight GB/s (% of B200 HBM peak); layer-chain tok/s"
QK = 256
BLOCK = {"q4_k": 144, "q6_k": 210}


def row_bytes(fmt, K):
    return K // QK * BLOCK[fmt]


# ----------------------------------------------------------------- workloads
def chain_layers(hidden, heads, kv_heads, head_dim, ffn, n_layers):
    """Per layer: (name, fmt, N, K, x-slot).  q|k|v share the attention input,
    gate|up share the FFN input; each is one fused launch over the stacked rows."""
    qkv = (heads + 2 * kv_heads) * head_dim
    mats = [("qkv", "q4_k", qkv, hidden, 0), ("o", "q4_k", hidden, heads * head_dim, 1),
            ("gate_up", "q4_k", 2 * ffn, hidden, 2), ("down", "q6_k", hidden, ffn, 3)]
    return [mats for _ in range(n_layers)]


WORKLOADS = {
    "llama8b_chain": dict(desc="Llama-3.1-8B-shaped decode chain, 32 layers, Q4_K + Q6_K down, batch 1",
                          layers=lambda: chain_layers(4096, 32, 8, 128, 14336, 32)),
    "gemv_q4k_4096": dict(desc="single Q4_K GEMV 4096 x 4096, batch 1 (64 distinct copies rotated)",
                          layers=lambda: [[("w", "q4_k", 4096, 4096, 0)] for _ in range(64)]),
    "gateup_q4k": dict(desc="Q4_K GEMV 28672 x 4096 (8B gate|up), 8 distinct copies rotated",
                       layers=lambda: [[("gate_up", "q4_k", 28672, 4096, 0)] for _ in range(8)]),
    "down_q6k": dict(desc="Q6_K GEMV 4096 x 14336 (8B down), 8 distinct copies rotated",
                     layers=lambda: [[("down", "q6_k", 4096, 14336, 0)] for _ in range(8)]),
}


def weight_bytes(layers):
    return sum(N * row_bytes(fmt, K) for mats in layers for (_, fmt, N, K, _) in mats)


# ------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi clock / throttle samples while the timed region runs."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except (FileNotFoundError, OSError):
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                mx = float(parts[1])
            except ValueError:
                continue
            for nm, v in zip(names, parts[3:7]):
                if v.lower() == "active":
                    reasons.add(nm)
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------ device setup
def build_device_chain(layers, seed, torch, kqgen, pinned_host=False):
    """Generate every weight matrix (host, parallel) and place it on the
    device; activation vectors per layer slot; output buffers."""
    dev_w, xs, ys = [], [], []
    for li, mats in enumerate(layers):
        wl, xl, yl = [], {}, []
        for mi, (name, fmt, N, K, slot) in enumerate(mats):
            host = np.empty(N * row_bytes(fmt, K), dtype=np.uint8)
            kqgen.matrix(fmt, kqgen.tensor_seed(seed, li, mi), N, K, out=host)
            t = torch.from_numpy(host)
            wl.append(t.pin_memory() if pinned_host else t.cuda())
            if slot not in xl:
                xh = torch.from_numpy(kqgen.normal_f32(kqgen.tensor_seed(seed ^ 0x5A5A, li, slot), K))
                xl[slot] = xh.cuda()
            yl.append(torch.empty(N, dtype=torch.float32, device="cuda"))
        torch.cuda.synchronize()
        dev_w.append(wl)
        xs.append(xl)
        ys.append(yl)
    return dev_w, xs, ys


def run_chain(kq, layers, dev_w, xs, ys, stream):
    for li, mats in enumerate(layers):
        for mi, (name, fmt, N, K, slot) in enumerate(mats):
            kq.gemv(dev_w[li][mi], fmt, N, K, xs[li][slot], ys[li][mi], stream=stream)


# --------------------------------------------------------------- the bench
def bench_kq(args, rank, world):
    import torch

    import kqgen
    from dequant_quant_gemv_b200 import kq

    torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", 0)))
    kq.lib()
    wl = WORKLOADS[args.workload]
    layers = wl["layers"]()
    wbytes = weight_bytes(layers)
    n_launch = sum(len(m) for m in layers)
    dev_w, xs, ys = build_device_chain(layers, 0xC0FFEE + 1 + rank, torch, kqgen)

    stream = torch.cuda.Stream()
    # every launch, graph replay and event of the bench goes to this stream
    torch.cuda.set_stream(stream)
    with torch.cuda.stream(stream):
        run_chain(kq, layers, dev_w, xs, ys, stream)  # sets kernel attributes before capture
    stream.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        run_chain(kq, layers, dev_w, xs, ys, stream)
    for _ in range(args.warmup):
        graph.replay()
    torch.cuda.synchronize()

    dist = world > 1
    if dist:
        import torch.distributed as tdist
        tdist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(torch.cuda.current_device()) as clk:
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(args.steps):
            graph.replay()
        e1.record(stream)
        torch.cuda.synchronize()
    ms = e0.elapsed_time(e1)
    if dist:
        t = torch.tensor([ms], device="cuda")
        tdist.all_reduce(t, op=tdist.ReduceOp.MAX)
        ms = float(t.item())
    ms_step = ms / args.steps
    gbs = wbytes * args.steps * world / (ms * 1e-3) / 1e9
    tok_s = args.steps * world / (ms * 1e-3)

    # dominant kernel: per-launch device time of each matrix kind, measured
    # with events on its own stream over all layers (weights never L2-hot)
    per_kind = {}
    kinds = sorted({m[0] for mats in layers for m in mats})
    for kind in kinds:
        idx = [(li, mi) for li, mats in enumerate(layers) for mi, m in enumerate(mats) if m[0] == kind]
        reps = max(1, 64 // len(idx))
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for _ in range(reps):
                for li, mi in idx:
                    name, fmt, N, K, slot = layers[li][mi]
                    kq.gemv(dev_w[li][mi], fmt, N, K, xs[li][slot], ys[li][mi], stream=stream)
        g.replay()
        torch.cuda.synchronize()
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            s0.record(stream)
            g.replay()
            s1.record(stream)
        torch.cuda.synchronize()
        del g
        n = reps * len(idx)
        t_us = s0.elapsed_time(s1) * 1e3 / n
        name, fmt, N, K, _ = layers[idx[0][0]][idx[0][1]]
        b = N * row_bytes(fmt, K)
        per_kind[kind] = dict(fmt=fmt, N=N, K=K, bytes=b, us=t_us, gbs=b / (t_us * 1e-6) / 1e9,
                              share=t_us * len(idx) / (ms_step * 1e3))
    dom = max(per_kind, key=lambda k: per_kind[k]["share"])

    # end to end through the public API with host buffers: activations in
    # from pinned memory, outputs back, every step
    x_host = [{s: t.cpu().pin_memory() for s, t in xl.items()} for xl in xs]
    y_host = [[torch.empty(t.numel(), dtype=torch.float32, pin_memory=True) for t in yl] for yl in ys]
    h2d = sum(t.numel() * 4 for xl in x_host for t in xl.values())
    d2h = sum(t.numel() * 4 for yl in y_host for t in yl)

    def e2e_step():
        for li, xl in enumerate(x_host):
            for s, t in xl.items():
                xs[li][s].copy_(t, non_blocking=True)
        graph.replay()
        for li, yl in enumerate(y_host):
            for mi, t in enumerate(yl):
                t.copy_(ys[li][mi], non_blocking=True)

    with torch.cuda.stream(stream):
        for _ in range(max(1, args.warmup)):
            e2e_step()
        torch.cuda.synchronize()
        if dist:
            tdist.barrier()
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record(stream)
        for _ in range(args.steps):
            e2e_step()
        f1.record(stream)
        torch.cuda.synchronize()
    ems = f0.elapsed_time(f1)
    if dist:
        t = torch.tensor([ems], device="cuda")
        tdist.all_reduce(t, op=tdist.ReduceOp.MAX)
        ems = float(t.item())
    e2e_gbs = wbytes * args.steps * world / (ems * 1e-3) / 1e9

    peaks = {}
    try:
        peaks = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))
    except (OSError, ValueError):
        pass
    hbm = peaks.get("hbm_gbs")
    peak_src = "measured" if hbm else "fallback"
    hbm = hbm or 6650.0
    dk = per_kind[dom]
    result = {
        "metric": METRIC, "value": round(gbs, 2), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_step, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32 (q4_k/q6_k weights)", "data": "synthetic",
        "tok_per_s": round(tok_s, 2), "frac_of_hbm_peak": round(gbs / world / hbm, 4),
        "config": {"workload": args.workload, "desc": wl["desc"], "weight_bytes_per_step": wbytes,
                   "launches_per_step": n_launch, "batch": 1, "parallelism": f"replicas{world}",
                   "l2": "inputs larger than L2 (no flush)" if wbytes > 2 * 126e6 else "rotating copies"},
        "roofline": {"bound": "hbm", "kernel": f"gemv_kernel<{dk['fmt']}> {dom} {dk['N']}x{dk['K']}",
                     "achieved": round(dk["gbs"], 1), "peak": hbm, "peak_source": peak_src, "unit": "GB/s",
                     "frac": round(dk["gbs"] / hbm, 4), "traffic": None},
        "kernels": {k: {kk: (round(vv, 4) if isinstance(vv, float) else vv) for kk, vv in v.items()}
                    for k, v in per_kind.items()},
        "e2e": {"value": round(e2e_gbs, 2), "unit": "GB/s", "tok_per_s": round(args.steps * world / (ems * 1e-3), 2),
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "clocks": clk.summary(),
        "gpu_launches": n_launch * args.steps,
    }
    return result


def cpu_baseline(args, budget_s=15.0):
    """The oracle as it stands, on a bounded sample of the same workload:
    a prefix of the chain's rows (every matrix kind), timed on all cores."""
    import kqgen
    import oracle

    layers = WORKLOADS[args.workload]["layers"]()
    cores = len(os.sched_getaffinity(0))
    done_bytes, t_total, rows_done = 0, 0.0, 0
    t_start = time.time()
    li = 0
    while time.time() - t_start < budget_s and li < len(layers):
        for mi, (name, fmt, N, K, slot) in enumerate(layers[li]):
            nrows = min(N, 512)
            W = kqgen.matrix(fmt, kqgen.tensor_seed(0xC0FFEE + 1, li, mi), nrows, K)
            x = kqgen.normal_f32(kqgen.tensor_seed((0xC0FFEE + 1) ^ 0x5A5A, li, slot), K)
            t0 = time.perf_counter()
            oracle.gemv(fmt, W, nrows, K, x, nthreads=cores)
            t_total += time.perf_counter() - t0
            done_bytes += nrows * row_bytes(fmt, K)
            rows_done += nrows
        li += 1
    gbs = done_bytes / t_total / 1e9
    wb = weight_bytes(layers)
    return {"value": round(gbs, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
            "tok_per_s": round(gbs * 1e9 / wb, 6),
            "sample": f"first {min(512, 4096)} rows of each matrix of {li} layer(s) ({rows_done} rows, "
                      f"{done_bytes / 1e6:.1f} MB), fp64 oracle, OpenMP over rows"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="llama8b_chain", choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="kq", choices=["kq", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))

    if args.impl == "reference":
        if rank != 0:
            return
        cb = cpu_baseline(args, budget_s=max(5.0, 2.0 * args.steps))
        line = {"metric": METRIC, "value": cb["value"], "unit": "GB/s", "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "f64", "data": "synthetic", "impl": "reference",
                "config": {"workload": args.workload, "desc": WORKLOADS[args.workload]["desc"]},
                "cpu_baseline": cb,
                "e2e": {"value": cb["value"], "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return

    if world > 1:
        import datetime

        import torch.distributed as tdist
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    result = bench_kq(args, rank, world)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(args)
    if rank == 0:
        print(json.dumps(result), flush=True)
    if world > 1:
        import torch.distributed as tdist
        tdist.destroy_process_group()


if __name__ == "__main__":
    main()
