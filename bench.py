#!/usr/bin/env python3
"""Benchmark of the fused K-quant dequant-GEMV path (libkq) on B200.

Default workload (the metric's configuration): the Llama-3.1-8B-shaped
decode chain at batch 1 -- per layer Wq|Wk|Wv (6144 x 4096), Wo
(4096 x 4096), Wgate|Wup (28672 x 4096) in Q4_K and Wdown (4096 x 14336) in
Q6_K, 32 layers, 4.41 GB of weights (larger than L2, so every step streams
the weights from HBM).  One step is one pass of the chain: 128 fused GEMV
launches replayed as one CUDA graph.  Metric: weight GB/s (algorithmic weight
bytes / time) and layer-chain tokens/s.

Other workloads (--workload): llama8b_layer_fused (the same chain with the
layer's RMSNorm and SiLU-gated product fused into the GEMVs), gemv_q4k_4096
(one 4096 x 4096 Q4_K GEMV),
verify8b_k{1,2,4,8} (the 8B chain with k activation columns),
moe30b (Qwen3-30B-A3B-shaped routed experts, top-8 of 128, 48 layers),
llama70b_resident / llama70b_stream (80-layer 70B-shaped chain in HBM, or
streamed from pinned host memory through 4 device slots), gateup_q4k and
down_q6k (single kernels, for profiling).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
  python bench.py --impl reference ...   # the CPU oracle on a bounded sample

Multi-GPU: the decode chain is one token's matvecs; ranks run independent
replicas (weak scaling) with no collective on the data path.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "K-quant dequant-GEMV weight GB/s (% of B200 HBM peak); layer-chain tok/s"
QK = 256
BLOCK = {"q4_k": 144, "q5_k": 176, "q6_k": 210, "q2_k": 84, "q3_k": 110, "q8_0": 272}  # bytes per 256 weights
SEED = 0xC0FFEE + 1


def row_bytes(fmt, K):
    return K // QK * BLOCK[fmt]


def dense_layer(hidden, heads, kv_heads, head_dim, ffn, fmt="q4_k", down_fmt="q6_k"):
    """(name, fmt, N, K, x-slot): q|k|v share the attention input, gate|up
    share the FFN input; each is one launch over the stacked rows.  `fmt`
    is the format of all but down, which is `down_fmt` (Q6_K in Q4_K_M and
    Q5_K_M files)."""
    qkv = (heads + 2 * kv_heads) * head_dim
    return [("qkv", fmt, qkv, hidden, 0), ("o", fmt, hidden, heads * head_dim, 1),
            ("gate_up", fmt, 2 * ffn, hidden, 2), ("down", down_fmt, hidden, ffn, 3)]


L8B = dict(hidden=4096, heads=32, kv_heads=8, head_dim=128, ffn=14336)
L70B = dict(hidden=8192, heads=64, kv_heads=8, head_dim=128, ffn=28672)
MOE30B = dict(hidden=2048, experts=128, top=8, ffn=768, layers=48)


def chain_spec(kind):
    if kind == "llama8b":
        return [dense_layer(**L8B) for _ in range(32)]
    if kind == "llama8b_q5k":
        return [dense_layer(**L8B, fmt="q5_k") for _ in range(32)]
    if kind == "llama8b_q2k":
        return [dense_layer(**L8B, fmt="q2_k", down_fmt="q3_k") for _ in range(32)]
    if kind == "llama8b_q3k":
        return [dense_layer(**L8B, fmt="q3_k", down_fmt="q4_k") for _ in range(32)]
    if kind == "llama8b_q80":
        return [dense_layer(**L8B, fmt="q8_0", down_fmt="q8_0") for _ in range(32)]
    if kind == "llama70b":
        return [dense_layer(**L70B) for _ in range(80)]
    if kind == "gemv_q4k_4096":
        return [[("w", "q4_k", 4096, 4096, 0)] for _ in range(64)]
    if kind == "gateup_q4k":
        return [[("gate_up", "q4_k", 28672, 4096, 0)] for _ in range(8)]
    if kind == "gateup_q5k":
        return [[("gate_up", "q5_k", 28672, 4096, 0)] for _ in range(8)]
    if kind == "gateup_q2k":
        return [[("gate_up", "q2_k", 28672, 4096, 0)] for _ in range(8)]
    if kind == "gateup_q3k":
        return [[("gate_up", "q3_k", 28672, 4096, 0)] for _ in range(8)]
    if kind == "gateup_q80":
        return [[("gate_up", "q8_0", 28672, 4096, 0)] for _ in range(8)]
    if kind == "down_q3k":
        return [[("down", "q3_k", 4096, 14336, 0)] for _ in range(8)]
    if kind == "down_q6k":
        return [[("down", "q6_k", 4096, 14336, 0)] for _ in range(8)]
    raise KeyError(kind)


WORKLOADS = {
    "llama8b_chain": "Llama-3.1-8B-shaped decode chain, 32 layers, Q4_K + Q6_K down, batch 1",
    "llama8b_q5k_chain": "Llama-3.1-8B-shaped decode chain with Q5_K qkv, o and gate|up and Q6_K down "
                         "(a Q5_K_M file's formats), 32 layers, batch 1",
    "verify8b_q5k_k8": "the Q5_K 8B-shaped chain, speculative-verify GEMV with k=8 activation columns",
    "gateup_q5k": "Q5_K GEMV 28672 x 4096 (8B gate|up), 8 distinct copies rotated",
    "llama8b_q2k_chain": "Llama-3.1-8B-shaped decode chain with Q2_K qkv, o and gate|up and Q3_K down, "
                         "32 layers, batch 1",
    "llama8b_q3k_chain": "Llama-3.1-8B-shaped decode chain with Q3_K qkv, o and gate|up and Q4_K down, "
                         "32 layers, batch 1",
    "gateup_q2k": "Q2_K GEMV 28672 x 4096 (8B gate|up), 8 distinct copies rotated",
    "gateup_q3k": "Q3_K GEMV 28672 x 4096 (8B gate|up), 8 distinct copies rotated",
    "down_q3k": "Q3_K GEMV 4096 x 14336 (8B down), 8 distinct copies rotated",
    "llama8b_q80_chain": "Llama-3.1-8B-shaped decode chain with every matrix in Q8_0, 32 layers, batch 1",
    "gateup_q80": "Q8_0 GEMV 28672 x 4096 (8B gate|up), 8 distinct copies rotated",
    "verify8b_q80_k8": "the Q8_0 8B-shaped chain, speculative-verify GEMV with k=8 activation columns",
    "verify8b_q2k_k8": "the Q2_K 8B-shaped chain (Q3_K down), speculative-verify GEMV with k=8 activation columns",
    "verify8b_q3k_k8": "the Q3_K 8B-shaped chain (Q4_K down), speculative-verify GEMV with k=8 activation columns",
    "llama8b_chain_steps": "the same chain through kq_gemv_steps (16 matvecs per persistent launch, each "
                           "waiting for the one before)",
    "llama8b_layer_fused": "the 8B-shaped chain with RMSNorm fused into qkv and gate|up and the SiLU-gated "
                           "product of gate|up's output fused into down",
    "llama8b_layer_fused_steps": "the fused-glue chain through kq_gemv_steps",
    "gemv_q4k_4096": "single Q4_K GEMV 4096 x 4096, batch 1 (64 distinct copies rotated)",
    "gateup_q4k": "Q4_K GEMV 28672 x 4096 (8B gate|up), 8 distinct copies rotated",
    "down_q6k": "Q6_K GEMV 4096 x 14336 (8B down), 8 distinct copies rotated",
    "verify8b_k1": "8B-shaped chain, speculative-verify GEMV with k=1 activation column",
    "verify8b_k2": "8B-shaped chain, speculative-verify GEMV with k=2 activation columns",
    "verify8b_k4": "8B-shaped chain, speculative-verify GEMV with k=4 activation columns",
    "verify8b_k8": "8B-shaped chain, speculative-verify GEMV with k=8 activation columns",
    "moe30b": "Qwen3-30B-A3B-shaped MoE GEMVs: 48 layers x 128 experts (gate|up 1536x2048, down 2048x768, "
              "Q4_K), top-8 routed ids per token, batch 1",
    "moe30b_stream": "the moe30b GEMVs with all experts in pinned host memory (16.3 GB): per token and layer "
                     "the 8 routed experts' gate|up and down copied to the device on demand (kq_moe_stream)",
    "llama70b_resident": "Llama-3.3-70B-shaped decode chain, 80 layers, Q4_K + Q6_K down, resident in HBM",
    "llama70b_resident_steps": "the 70B-shaped resident chain through kq_gemv_steps",
    "llama70b_stream": "Llama-3.3-70B-shaped decode chain, 80 layers, weights in pinned host memory streamed "
                       "through 4 device layer slots",
    "llama70b_stream_20gb": "the streamed 70B-shaped chain within a 20 GB device budget: the leading layers that "
                            "fit stay resident beside 4 slots, the rest stream (kq_chain_plan)",
}


# ------------------------------------------------------------------- clocks
class ClockSampler:
    """SM clock, power and throttle-reason samples taken while the timed
    region runs: NVML polled every millisecond from a thread (nvidia-smi at
    50 ms if NVML is missing).  Only samples between start() and stop() --
    the timed region -- are kept."""

    REASONS = {"hw_slowdown": 0x8, "hw_thermal_slowdown": 0x40, "sw_thermal_slowdown": 0x20, "sw_power_cap": 0x4}

    def __init__(self, index):
        self.index = index
        self.samples = []
        self.active = False
        self.done = False
        self.mx = None
        self.nvml = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nvml = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.mx = float(pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM))
        except Exception:
            self.nvml = None

    def _sample_nvml(self):
        n = self.nvml
        try:
            fn = getattr(n, "nvmlDeviceGetCurrentClocksEventReasons", None) or n.nvmlDeviceGetCurrentClocksThrottleReasons
            return (float(n.nvmlDeviceGetClockInfo(self.h, n.NVML_CLOCK_SM)),
                    n.nvmlDeviceGetPowerUsage(self.h) / 1000.0, int(fn(self.h)))
        except Exception:
            return None

    def _loop(self):
        while not self.done:
            if self.active:
                smp = self._sample_nvml()
                if smp is not None:
                    self.samples.append(smp)
            time.sleep(0.001)

    def _smi_loop(self):
        fields = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
                  "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
                  "clocks_event_reasons.sw_power_cap")
        try:
            proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={fields}",
                                     "--format=csv,noheader,nounits", "-lms", "50"],
                                    stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (FileNotFoundError, OSError):
            return
        self.proc = proc
        for line in proc.stdout:
            if not self.active:
                continue
            parts = [p.strip() for p in line.split(",")]
            try:
                bits = sum(v for (nm, v), st in zip(self.REASONS.items(), parts[3:7]) if st.lower() == "active")
                self.mx = float(parts[1])
                self.samples.append((float(parts[0]), float(parts[2]), bits))
            except (ValueError, IndexError):
                continue

    def __enter__(self):
        self.proc = None
        self.t = threading.Thread(target=self._loop if self.nvml else self._smi_loop, daemon=True)
        self.t.start()
        return self

    def start(self):
        self.active = True

    def stop(self):
        self.active = False

    def __exit__(self, *exc):
        self.done = True
        self.active = False
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        self.t.join(timeout=5)

    def summary(self):
        sm = [a for a, _, _ in self.samples]
        pw = [b for _, b, _ in self.samples]
        reasons = sorted(nm for nm, bit in self.REASONS.items() if any(r & bit for _, _, r in self.samples))
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": self.mx,
                "power_w_max": max(pw) if pw else None, "reasons": reasons, "samples": len(sm),
                "source": "nvml, 1 ms" if self.nvml else "nvidia-smi, 50 ms"}


# --------------------------------------------------------------- workloads
class Resident:
    """A chain of fused GEMV launches over weights resident in HBM.

    Activations of all matrices live in one device buffer (and one pinned
    host buffer for the end-to-end leg), outputs likewise."""

    graphable = True

    def __init__(self, torch, kq, kqgen, spec, seed, k=1, steps=False):
        self.torch, self.kq, self.spec, self.k = torch, kq, spec, k
        self.use_steps = steps
        self.launches = [(li, mi) for li, mats in enumerate(spec) for mi in range(len(mats))]
        self.weight_bytes = sum(N * row_bytes(f, K) for mats in spec for (_, f, N, K, _) in mats)
        # activations: one slot per (layer, x-slot), k columns each
        xoff, yoff, self.xslot, self.yslot = 0, 0, {}, {}
        for li, mats in enumerate(spec):
            for mi, (_, f, N, K, slot) in enumerate(mats):
                if slot is not None and (li, slot) not in self.xslot:
                    self.xslot[(li, slot)] = (xoff, K)
                    xoff += k * K
                self.yslot[(li, mi)] = (yoff, N)
                yoff += k * N
        self.X = torch.empty(xoff, dtype=torch.float32, device="cuda")
        self.Y = torch.empty(yoff, dtype=torch.float32, device="cuda")
        xh = np.empty(xoff, np.float32)
        for (li, slot), (off, K) in self.xslot.items():
            kqgen.normal_f32(kqgen.tensor_seed(seed ^ 0x5A5A, li, slot), k * K, out=xh[off:off + k * K])
        self.X.copy_(torch.from_numpy(xh))
        self.W = []
        for li, mats in enumerate(spec):
            row = []
            for mi, (_, f, N, K, _) in enumerate(mats):
                host = np.empty(N * row_bytes(f, K), np.uint8)
                kqgen.matrix(f, kqgen.tensor_seed(seed, li, mi), N, K, out=host)
                row.append(torch.from_numpy(host).cuda())
            self.W.append(row)
        torch.cuda.synchronize()
        if steps:
            self.build_steps()

    # ---- the chain as one list of steps (kq_gemv_steps)
    def step_args(self, li, mi):
        """(x, prologue kind, gamma) of matrix mi of layer li."""
        return self.x_of(li, mi)[0], "none", None

    def build_steps(self):
        """Every matrix of the chain as a step of kq_gemv_steps, each marked
        `after`: as in decode, a step starts only when the step before it has
        finished on the whole GPU (the launches-per-matrix order)."""
        self.steps, self.kind_steps = [], {}
        for li, mi in self.launches:
            name, f, N, K, _ = self.spec[li][mi]
            x, kind, gamma = self.step_args(li, mi)
            st = self.kq.make_step(self.W[li][mi], f, N, K, x, self.y_of(li, mi)[0], kind, gamma, 1e-5, after=True)
            self.steps.append(st)
            self.kind_steps.setdefault(name, []).append(st)
        self.launches_per_step = -(-len(self.steps) // 16)

    def launch_kind(self, name, stream):
        self.kq.gemv_steps(self.kind_steps[name], stream=stream)

    def x_of(self, li, mi):
        off, K = self.xslot[(li, self.spec[li][mi][4])]
        return self.X[off:off + self.k * K].view(self.k, K)

    def y_of(self, li, mi):
        off, N = self.yslot[(li, mi)]
        return self.Y[off:off + self.k * N].view(self.k, N)

    def launch(self, li, mi, stream):
        _, f, N, K, _ = self.spec[li][mi]
        if self.k == 1:
            self.kq.gemv(self.W[li][mi], f, N, K, self.x_of(li, mi)[0], self.y_of(li, mi)[0], stream=stream)
        else:
            self.kq.gemv_multi(self.W[li][mi], f, N, K, self.x_of(li, mi), self.y_of(li, mi), stream=stream)

    def step(self, stream):
        if self.use_steps:
            self.kq.gemv_steps(self.steps, stream=stream)
            return
        for li, mi in self.launches:
            self.launch(li, mi, stream)

    def kinds(self):
        out = {}
        for li, mi in self.launches:
            name, f, N, K, _ = self.spec[li][mi]
            out.setdefault(name, dict(fmt=f, N=N, K=K, bytes=N * row_bytes(f, K), launches=[]))
            out[name]["launches"].append((li, mi))
        return out

    def io(self):
        return [self.X], [self.Y]

    def layer_io(self):
        """Per layer: (x offset, x length, y offset, y length) in elements
        of X and Y (each layer's slots are contiguous, in layer order)."""
        out = []
        for li, mats in enumerate(self.spec):
            xs = [self.xslot[(li, slot)] for (_, _, _, _, slot) in mats if slot is not None]
            ys = [self.yslot[(li, mi)] for mi in range(len(mats))]
            x0 = min(o for o, _ in xs)
            x1 = max(o + self.k * K for o, K in xs)
            y0 = min(o for o, _ in ys)
            y1 = max(o + self.k * N for o, N in ys)
            out.append((x0, x1 - x0, y0, y1 - y0))
        return out


class FusedLayer(Resident):
    """The 8B chain with the decode layer's glue inside the GEMVs: qkv and
    gate|up normalise their input (RMSNorm, per-layer weights), and down
    takes gate|up's output [g; u] directly through the SiLU-gated prologue,
    so the layer needs no separate norm or activation kernel.  Attention and
    the residual adds are not on this path: o and each layer's norm inputs
    keep their own seeded activations."""

    EPS = 1e-5

    def __init__(self, torch, kq, kqgen, spec, seed, steps=False):
        fused = [[m if m[0] != "down" else m[:4] + (None,) for m in mats] for mats in spec]
        super().__init__(torch, kq, kqgen, fused, seed)
        self.gu = {li: mi for li, mats in enumerate(fused) for mi, m in enumerate(mats) if m[0] == "gate_up"}
        n = len(fused)
        K = fused[0][0][3]
        g = 1.0 + 0.1 * kqgen.normal_f32(seed ^ 0x6A3, 2 * n * K).astype(np.float32)
        self.gamma = torch.from_numpy(g).cuda().view(n, 2, K)
        torch.cuda.synchronize()
        self.use_steps = steps
        if steps:
            self.build_steps()

    def step_args(self, li, mi):
        name = self.spec[li][mi][0]
        if name == "qkv" or name == "gate_up":
            return self.x_of(li, mi)[0], "rmsnorm", self.gamma[li, 0 if name == "qkv" else 1]
        if name == "down":
            return self.y_of(li, self.gu[li])[0], "swiglu", None
        return self.x_of(li, mi)[0], "none", None

    def launch(self, li, mi, stream):
        name, f, N, K, _ = self.spec[li][mi]
        W, y = self.W[li][mi], self.y_of(li, mi)[0]
        if name == "qkv" or name == "gate_up":
            self.kq.gemv_fused(W, f, N, K, self.x_of(li, mi)[0], "rmsnorm",
                               self.gamma[li, 0 if name == "qkv" else 1], self.EPS, Y=y, stream=stream)
        elif name == "down":
            self.kq.gemv_fused(W, f, N, K, self.y_of(li, self.gu[li])[0], "swiglu", Y=y, stream=stream)
        else:
            self.kq.gemv(W, f, N, K, self.x_of(li, mi)[0], y, stream=stream)


class MoE:
    """Routed-expert GEMVs: per layer one launch for the routed experts'
    gate|up rows (shared x) and one for their down rows (one x per id)."""

    graphable = True

    def __init__(self, torch, kq, kqgen, seed, tokens=4):
        c = MOE30B
        self.torch, self.kq = torch, kq
        H, E, top, F, Lyr = c["hidden"], c["experts"], c["top"], c["ffn"], c["layers"]
        self.E, self.top, self.H, self.F, self.L = E, top, H, F, Lyr
        self.gu_stride = 2 * F * row_bytes("q4_k", H)
        self.dn_stride = H * row_bytes("q4_k", F)
        self.weight_bytes = Lyr * top * (self.gu_stride + self.dn_stride)
        self.Wgu, self.Wdn = [], []
        for l in range(Lyr):
            h = np.empty(E * self.gu_stride, np.uint8)
            kqgen.matrix("q4_k", kqgen.tensor_seed(seed, l, 0), E * 2 * F, H, out=h)
            self.Wgu.append(torch.from_numpy(h).cuda())
            h = np.empty(E * self.dn_stride, np.uint8)
            kqgen.matrix("q4_k", kqgen.tensor_seed(seed, l, 1), E * H, F, out=h)
            self.Wdn.append(torch.from_numpy(h).cuda())
        # routed ids for `tokens` tokens; the step copies the next token's ids
        # into the buffer the kernels read (as a router would write them)
        ids = np.stack([np.stack([kqgen.topk_ids(kqgen.tensor_seed(seed ^ 0x1D5, t, l), E, top)
                                  for l in range(Lyr)]) for t in range(tokens)])
        self.ids_all = torch.from_numpy(ids).cuda()               # (tokens, L, top)
        self.ids = torch.empty((Lyr, top), dtype=torch.int32, device="cuda")
        self.t = 0
        self.X = torch.from_numpy(kqgen.normal_f32(seed ^ 0x77, Lyr * H + Lyr * top * F)).cuda()
        self.Y = torch.empty(Lyr * top * 2 * F + Lyr * top * H, dtype=torch.float32, device="cuda")
        self.status = torch.zeros(1, dtype=torch.int32, device="cuda")
        self.launches = [(l, j) for l in range(Lyr) for j in range(2)]
        torch.cuda.synchronize()

    def xg(self, l):
        return self.X[l * self.H:(l + 1) * self.H]

    def xd(self, l):
        o = self.L * self.H + l * self.top * self.F
        return self.X[o:o + self.top * self.F].view(self.top, self.F)

    def yg(self, l):
        o = l * self.top * 2 * self.F
        return self.Y[o:o + self.top * 2 * self.F].view(self.top, 2 * self.F)

    def yd(self, l):
        o = self.L * self.top * 2 * self.F + l * self.top * self.H
        return self.Y[o:o + self.top * self.H].view(self.top, self.H)

    def launch(self, l, j, stream):
        kq = self.kq
        if j == 0:
            kq.moe_gemv(self.Wgu[l], "q4_k", self.E, 2 * self.F, self.H, self.ids[l], self.xg(l), self.yg(l),
                        status=self.status, expert_stride=self.gu_stride, stream=stream)
        else:
            kq.moe_gemv(self.Wdn[l], "q4_k", self.E, self.H, self.F, self.ids[l], self.xd(l), self.yd(l),
                        status=self.status, expert_stride=self.dn_stride, stream=stream)

    def step(self, stream):
        for l, j in self.launches:
            self.launch(l, j, stream)

    def advance(self):
        self.ids.copy_(self.ids_all[self.t % self.ids_all.shape[0]], non_blocking=True)
        self.t += 1

    def kinds(self):
        return {"moe_gate_up": dict(fmt="q4_k", N=2 * self.F, K=self.H, bytes=self.top * self.gu_stride,
                                    launches=[(l, 0) for l in range(self.L)]),
                "moe_down": dict(fmt="q4_k", N=self.H, K=self.F, bytes=self.top * self.dn_stride,
                                 launches=[(l, 1) for l in range(self.L)])}

    def io(self):
        return [self.X], [self.Y]


class Streamed:
    """The chain with its weights in pinned host memory (kq_chain)."""

    graphable = False

    def __init__(self, torch, kq, kqgen, spec, seed, n_slots=4, budget=None):
        self.torch, self.kq, self.spec = torch, kq, spec
        self.weight_bytes = sum(N * row_bytes(f, K) for mats in spec for (_, f, N, K, _) in mats)
        # one host buffer for every weight, page-locked in place (the torch
        # pinned allocator would round each tensor up to a power of two)
        self.host = np.empty(self.weight_bytes, np.uint8)
        mats, xs, ys, off = [], [], [], 0
        for li, layer in enumerate(spec):
            row = []
            for mi, (_, f, N, K, _) in enumerate(layer):
                nb = N * row_bytes(f, K)
                view = self.host[off:off + nb]
                kqgen.matrix(f, kqgen.tensor_seed(seed, li, mi), N, K, out=view)
                row.append((torch.from_numpy(view), f, N, K))
                off += nb
            mats.append(row)
        rc = torch.cuda.cudart().cudaHostRegister(self.host.ctypes.data, self.host.nbytes, 0)
        if int(rc) != 0:
            raise RuntimeError(f"cudaHostRegister failed ({rc})")
        self.X = torch.from_numpy(kqgen.normal_f32(seed ^ 0x5A5A, sum(m[3] for r in mats for m in r))).cuda()
        self.Y = torch.empty(sum(m[2] for r in mats for m in r), dtype=torch.float32, device="cuda")
        xo = yo = 0
        for r in mats:
            for (_, f, N, K) in r:
                xs.append(self.X[xo:xo + K])
                ys.append(self.Y[yo:yo + N])
                xo += K
                yo += N
        self.xs, self.ys = xs, ys
        # with a device-memory budget: the leading layers that fit stay
        # resident (kq_chain_plan), the rest stream
        self.n_resident = 0
        if budget is not None:
            self.n_resident, n_slots = kq.chain_plan([[(None, f, N, K) for (_, f, N, K) in r] for r in mats], budget,
                                                     max_slots=n_slots)
        self.streamed_bytes = sum(N * row_bytes(f, K) for li, r in enumerate(mats) for (_, f, N, K) in r
                                  if li >= self.n_resident)
        self.chain = kq.Chain(mats, n_slots=n_slots, n_resident=self.n_resident)
        self.launches = [None] * sum(len(r) for r in mats)

    def step(self, stream):
        self.chain.run(self.xs, self.ys, stream=stream)

    def kinds(self):
        return {}

    def io(self):
        return [self.X], [self.Y]


class MoEStreamed(MoE):
    """The MoE GEMVs with every expert in pinned host memory: per layer and
    token the 8 routed experts' gate|up and down matrices are copied to the
    device on demand (kq_moe_stream) and the routed GEMVs read the copies."""

    graphable = False

    def __init__(self, torch, kq, kqgen, seed, tokens=4):
        c = MOE30B
        self.torch, self.kq = torch, kq
        H, E, top, F, Lyr = c["hidden"], c["experts"], c["top"], c["ffn"], c["layers"]
        self.E, self.top, self.H, self.F, self.L = E, top, H, F, Lyr
        self.gu_stride = 2 * F * row_bytes("q4_k", H)
        self.dn_stride = H * row_bytes("q4_k", F)
        self.weight_bytes = Lyr * top * (self.gu_stride + self.dn_stride)
        self.streamed_bytes = self.weight_bytes
        self.n_resident = 0
        # every layer's experts in one host stack per matrix kind (expert
        # l*E + e is expert e of layer l), page-locked in place
        self.hgu = np.empty(Lyr * E * self.gu_stride, np.uint8)
        self.hdn = np.empty(Lyr * E * self.dn_stride, np.uint8)
        for l in range(Lyr):
            kqgen.matrix("q4_k", kqgen.tensor_seed(seed, l, 0), E * 2 * F, H,
                         out=self.hgu[l * E * self.gu_stride:(l + 1) * E * self.gu_stride])
            kqgen.matrix("q4_k", kqgen.tensor_seed(seed, l, 1), E * H, F,
                         out=self.hdn[l * E * self.dn_stride:(l + 1) * E * self.dn_stride])
        for h in (self.hgu, self.hdn):
            rc = torch.cuda.cudart().cudaHostRegister(h.ctypes.data, h.nbytes, 0)
            if int(rc) != 0:
                raise RuntimeError(f"cudaHostRegister failed ({rc})")
        self.msgu = kq.MoEStream(torch.from_numpy(self.hgu), "q4_k", Lyr * E, 2 * F, H, max_ids=top, n_sets=2)
        self.msdn = kq.MoEStream(torch.from_numpy(self.hdn), "q4_k", Lyr * E, H, F, max_ids=top, n_sets=2)
        self.ids_all = np.stack([np.stack([kqgen.topk_ids(kqgen.tensor_seed(seed ^ 0x1D5, t, l), E, top) + l * E
                                           for l in range(Lyr)]) for t in range(tokens)]).astype(np.int32)
        self.t = 0
        self.X = torch.from_numpy(kqgen.normal_f32(seed ^ 0x77, Lyr * H + Lyr * top * F)).cuda()
        self.Y = torch.empty(Lyr * top * 2 * F + Lyr * top * H, dtype=torch.float32, device="cuda")
        self.launches = [(l, j) for l in range(Lyr) for j in range(2)]
        torch.cuda.synchronize()

    def launch(self, l, j, stream):
        ids = self.ids_all[self.t % self.ids_all.shape[0], l]
        if j == 0:
            self.msgu.run(ids, self.xg(l), 0, self.yg(l), stream=stream)
        else:
            self.msdn.run(ids, self.xd(l), self.F, self.yd(l), stream=stream)

    def advance(self):
        self.t += 1

    def kinds(self):
        return {}


CHAIN_BASE = {"llama8b_chain": "llama8b", "llama8b_chain_steps": "llama8b", "llama8b_layer_fused": "llama8b",
              "llama8b_layer_fused_steps": "llama8b", "llama8b_q5k_chain": "llama8b_q5k",
              "verify8b_q5k_k8": "llama8b_q5k", "verify8b_q80_k8": "llama8b_q80", "verify8b_q2k_k8": "llama8b_q2k", "verify8b_q3k_k8": "llama8b_q3k",
              "llama8b_q2k_chain": "llama8b_q2k",
              "llama8b_q3k_chain": "llama8b_q3k", "llama8b_q80_chain": "llama8b_q80",
              "llama70b_resident": "llama70b", "llama70b_resident_steps": "llama70b",
              "llama70b_stream": "llama70b", "llama70b_stream_20gb": "llama70b"}


def workload_spec(name):
    """(spec, columns) of a chain-shaped workload, or (None, 1) for MoE."""
    if name in ("moe30b", "moe30b_stream"):
        return None, 1
    if name.startswith("verify8b_k"):
        return chain_spec("llama8b"), int(name[len("verify8b_k"):])
    k = 8 if name in ("verify8b_q5k_k8", "verify8b_q80_k8", "verify8b_q2k_k8", "verify8b_q3k_k8") else 1
    return chain_spec(CHAIN_BASE.get(name, name)), k


def workload_config(name, world):
    """The `config` of the JSON line, computed on the host from the shapes
    alone, so that both arms (the GPU path and the oracle) report the same
    keys and values."""
    spec, k = workload_spec(name)
    if spec is None:
        c = MOE30B
        weight_bytes = c["layers"] * c["top"] * (2 * c["ffn"] * row_bytes("q4_k", c["hidden"])
                                                + c["hidden"] * row_bytes("q4_k", c["ffn"]))
        launches = 2 * c["layers"]
    else:
        weight_bytes = sum(N * row_bytes(f, K) for mats in spec for (_, f, N, K, _) in mats)
        launches = sum(len(m) for m in spec)
        if name.endswith("_steps"):
            launches = -(-launches // 16)
    return {"workload": name, "desc": WORKLOADS[name], "weight_bytes_per_step": weight_bytes,
            "launches_per_step": launches, "columns": k, "batch": 1, "parallelism": f"replicas{world}",
            "l2": "inputs larger than L2 (no flush)" if weight_bytes > 2 * 126e6 else "rotating copies"}


def dtype_of(name):
    """The arithmetic the path computes in (fp32 accumulation throughout)."""
    spec, k = workload_spec(name)
    if k == 1:
        return "f32 acc; activations int14 per group of 32, exact int32 sub-block sums (DP4A)"
    return "f32 acc; exact fp16 weight operands x fp16 activations (one term per column and super-block scale), tensor cores"


def make_workload(name, torch, kq, kqgen, seed):
    if name in ("llama8b_chain", "llama8b_chain_steps"):
        return Resident(torch, kq, kqgen, chain_spec("llama8b"), seed, steps=name.endswith("_steps"))
    if name in ("llama8b_layer_fused", "llama8b_layer_fused_steps"):
        return FusedLayer(torch, kq, kqgen, chain_spec("llama8b"), seed, steps=name.endswith("_steps"))
    if name == "llama8b_q5k_chain":
        return Resident(torch, kq, kqgen, chain_spec("llama8b_q5k"), seed)
    if name == "verify8b_q5k_k8":
        return Resident(torch, kq, kqgen, chain_spec("llama8b_q5k"), seed, k=8)
    if name in ("verify8b_q80_k8", "verify8b_q2k_k8", "verify8b_q3k_k8"):
        return Resident(torch, kq, kqgen, chain_spec(CHAIN_BASE[name]), seed, k=8)
    if name in ("llama8b_q2k_chain", "llama8b_q3k_chain", "llama8b_q80_chain"):
        return Resident(torch, kq, kqgen, chain_spec(name[:-len("_chain")]), seed)
    if name in ("gemv_q4k_4096", "gateup_q4k", "gateup_q5k", "down_q6k", "gateup_q2k", "gateup_q3k", "down_q3k",
                "gateup_q80"):
        return Resident(torch, kq, kqgen, chain_spec(name), seed)
    if name.startswith("verify8b_k"):
        k = int(name[len("verify8b_k"):])
        return Resident(torch, kq, kqgen, chain_spec("llama8b"), seed, k=k)
    if name == "moe30b":
        return MoE(torch, kq, kqgen, seed)
    if name == "moe30b_stream":
        return MoEStreamed(torch, kq, kqgen, seed)
    if name in ("llama70b_resident", "llama70b_resident_steps"):
        return Resident(torch, kq, kqgen, chain_spec("llama70b"), seed, steps=name.endswith("_steps"))
    if name == "llama70b_stream":
        return Streamed(torch, kq, kqgen, chain_spec("llama70b"), seed)
    if name == "llama70b_stream_20gb":
        return Streamed(torch, kq, kqgen, chain_spec("llama70b"), seed, budget=20 * 10**9)
    raise KeyError(name)


def h2d_peak_gbs(torch, nbytes=512 << 20, reps=5):
    """Pinned host -> device copy bandwidth (the streamed chain's roofline)."""
    h = torch.empty(nbytes, dtype=torch.uint8, pin_memory=True)
    d = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    d.copy_(h, non_blocking=True)
    torch.cuda.synchronize()
    best = 0.0
    for _ in range(reps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        d.copy_(h, non_blocking=True)
        e1.record()
        torch.cuda.synchronize()
        best = max(best, nbytes / (e0.elapsed_time(e1) * 1e-3) / 1e9)
    del h, d
    return best


def read_roofline(torch, kq, nbytes=2 << 30, reps=5):
    """Read-only HBM bandwidth (GB/s) of a 2 GiB buffer read once, best of
    `reps`, by the two probes of kq_read_probe: 16-byte loads from a full
    grid, and the GEMV kernels' own bulk-copy ring with no work per stage."""
    buf = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    buf.random_(0, 255)
    out = torch.zeros(1, dtype=torch.int32, device="cuda")
    res = {}
    for mode, name in ((0, "loads"), (1, "bulk_ring")):
        kq.read_probe(buf, mode, out)
        torch.cuda.synchronize()
        best = 0.0
        for _ in range(reps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            kq.read_probe(buf, mode, out)
            e1.record()
            torch.cuda.synchronize()
            best = max(best, nbytes / (e0.elapsed_time(e1) * 1e-3) / 1e9)
        res[name] = round(best, 1)
    del buf
    return res


# -------------------------------------------------- measured DRAM traffic
# dram__bytes_read.sum + dram__bytes_write.sum per launch of the dominant
# kernel, from one ncu capture (the summaries and commands are kept with
# the profiles), keyed by (format, N, K, columns).  Valid only for the kernel sources they
# were taken on: any change to the code in csrc/ (comments aside) changes the
# hash and the bench reports traffic as null until the counters are taken
# again.
TRAFFIC_SOURCES = "095a363cf2eb3a5f"
TRAFFIC = {
    # gemv1_kernel (single column, DP4A): the 8B-shaped chain's matrices
    ("q4_k", 6144, 4096, 1): 14_215_720 + 16,
    ("q4_k", 4096, 4096, 1): 9_497_536,
    ("q4_k", 28672, 4096, 1): 66_120_672 + 3_008,
    ("q6_k", 4096, 14336, 1): 48_288_880 + 1_136,
    # mma_kernel (tensor cores), 8 columns
    ("q4_k", 6144, 4096, 8): 14_337_792,
    ("q4_k", 4096, 4096, 8): 9_618_944,
    ("q4_k", 28672, 4096, 8): 66_243_840 + 1_024,
    ("q6_k", 4096, 14336, 8): 48_682_240,
}


def _code_only(src: str) -> str:
    """C++ source without its comments and with whitespace collapsed, so
    that an edit of comments alone keeps the hash (string literals holding
    comment markers do not occur in these sources)."""
    src = re.sub(r"/\*.*?\*/", " ", src, flags=re.S)
    src = re.sub(r"//[^\n]*", " ", src)
    return " ".join(src.split())


def kernel_sources_hash():
    """Hash of the kernel sources' code (comments and layout ignored)."""
    h = hashlib.sha256()
    d = os.path.join(ROOT, "dequant_quant_gemv_b200", "csrc")
    for n in sorted(os.listdir(d)):
        if n.endswith((".cu", ".cuh", ".h")):
            h.update(n.encode())
            with open(os.path.join(d, n), encoding="utf-8") as f:
                h.update(_code_only(f.read()).encode())
    return h.hexdigest()[:16]


def measured_traffic(fmt, N, K, k):
    if kernel_sources_hash() != TRAFFIC_SOURCES:
        return None
    return TRAFFIC.get((fmt, N, K, k))


# ------------------------------------------------------ replicas over ranks
def rank_seed(rank):
    """Each rank decodes its own replica: same shapes, its own weights and
    activations."""
    return SEED + rank


def max_over_ranks(value, device):
    """The largest `value` over all ranks (the slowest replica's time); the
    process group's own backend does the reduction (NCCL on GPUs, gloo on
    CPU)."""
    import torch
    import torch.distributed as tdist

    if not (tdist.is_available() and tdist.is_initialized()) or tdist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    tdist.all_reduce(t, op=tdist.ReduceOp.MAX)
    return float(t.item())


def job_rate(units_per_rank_step, steps, world, ms_max):
    """Whole-job rate: the units every rank processed over the slowest
    rank's time (weak scaling, each rank a full replica)."""
    return units_per_rank_step * steps * world / (ms_max * 1e-3)


# --------------------------------------------------------------- the bench
def bench_kq(args, rank, world):
    import torch

    import kqgen
    from dequant_quant_gemv_b200 import kq

    torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", 0)))
    kq.lib()
    dist = world > 1
    if dist:
        import torch.distributed as tdist
    wl = make_workload(args.workload, torch, kq, kqgen, rank_seed(rank))
    stream = torch.cuda.Stream()
    torch.cuda.set_stream(stream)   # every launch, replay and event goes here
    advance = getattr(wl, "advance", None)

    def one_step():
        if advance:
            advance()
        wl.step(stream)

    one_step()                       # sets kernel attributes before any capture
    torch.cuda.synchronize()
    if wl.graphable:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            wl.step(stream)

        def run_step():
            if advance:
                advance()
            graph.replay()
    else:
        run_step = one_step
    for _ in range(args.warmup):
        run_step()
    torch.cuda.synchronize()
    if dist:
        tdist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(torch.cuda.current_device()) as clk:
        torch.cuda.synchronize()
        clk.start()
        e0.record(stream)
        for _ in range(args.steps):
            run_step()
        e1.record(stream)
        # poll (releasing the interpreter lock) so that the clock thread
        # keeps sampling until the timed work has finished
        while not e1.query():
            time.sleep(0.0002)
        torch.cuda.synchronize()
        clk.stop()
    ms = max_over_ranks(e0.elapsed_time(e1), "cuda")
    ms_step = ms / args.steps
    k = getattr(wl, "k", 1)
    gbs = job_rate(wl.weight_bytes, args.steps, world, ms) / 1e9
    tok_s = job_rate(k, args.steps, world, ms)

    # per-kernel device time of each matrix kind: a graph of all its
    # launches (different layers' weights, so never L2-hot), events around it
    per_kind = {}
    if wl.graphable:
        for name, kd in wl.kinds().items():
            reps = max(1, 64 // len(kd["launches"]))
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                for _ in range(reps):
                    if getattr(wl, "use_steps", False):
                        wl.launch_kind(name, stream)
                    else:
                        for (a, b) in kd["launches"]:
                            wl.launch(a, b, stream)
            g.replay()
            torch.cuda.synchronize()
            s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            s0.record(stream)
            g.replay()
            s1.record(stream)
            torch.cuda.synchronize()
            n = reps * len(kd["launches"])
            t_us = s0.elapsed_time(s1) * 1e3 / n
            per_kind[name] = dict(fmt=kd["fmt"], N=kd["N"], K=kd["K"], bytes=kd["bytes"], us=round(t_us, 3),
                                  gbs=round(kd["bytes"] / (t_us * 1e-6) / 1e9, 1),
                                  share=round(t_us * len(kd["launches"]) / (ms_step * 1e3), 4))
            del g

    # end to end through the public API with host buffers: the step's
    # activations in from pinned memory and its outputs back, every step
    xin, yout = wl.io()
    xh = [t.cpu().pin_memory() for t in xin]
    yh = [torch.empty(t.numel(), dtype=t.dtype, pin_memory=True) for t in yout]
    h2d = sum(t.numel() * t.element_size() for t in xh)
    d2h = sum(t.numel() * t.element_size() for t in yh)

    def e2e_step():
        for d, h in zip(xin, xh):
            d.copy_(h, non_blocking=True)
        run_step()
        for h, d in zip(yh, yout):
            h.copy_(d, non_blocking=True)

    if isinstance(wl, Resident) and not wl.use_steps:
        # the decode chain: the activations come in on a copy stream while
        # earlier layers compute, and the outputs go back on another once
        # their launches are done (one graph per step).  A launch that waits
        # for a copy loses its programmatic overlap with the launch before
        # it (1.5-4 us measured per wait), so the copies go in a few
        # chunks that grow fourfold: inputs of layer 0, of the next 3, the
        # next 12, then the rest (each chunk copied while the layers before
        # it compute, a layer's compute taking ~15x its copy); outputs in
        # the mirrored chunks, the last layer's alone (the one copy left
        # exposed after the last launch).
        cs_in, cs_out = torch.cuda.Stream(), torch.cuda.Stream()
        X, Y, XH, YH = xin[0], yout[0], xh[0], yh[0]
        lio = wl.layer_io()
        nl = len(lio)

        sizes, left = [], nl
        for n in (1, 3, 12):
            if left > n:
                sizes.append(n)
                left -= n
        sizes.append(left)

        def spans(sz):
            out, i = [], 0
            for n in sz:
                out.append((i, i + n - 1))
                i += n
            return out

        in_chunks = spans(sizes)
        out_chunks = spans(sizes[::-1])
        g_e2e = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_e2e, stream=stream):
            fork = torch.cuda.Event()
            fork.record(stream)
            cs_in.wait_event(fork)
            cs_out.wait_event(fork)
            ev_in = {}
            for (a, b) in in_chunks:
                x0, x1 = lio[a][0], lio[b][0] + lio[b][1]
                with torch.cuda.stream(cs_in):
                    X[x0:x1].copy_(XH[x0:x1], non_blocking=True)
                    e = torch.cuda.Event()
                    e.record(cs_in)
                ev_in[a] = e
            out_last = {b: a for (a, b) in out_chunks}
            for li in range(nl):
                if li in ev_in:
                    stream.wait_event(ev_in[li])
                for mi in range(len(wl.spec[li])):
                    wl.launch(li, mi, stream)
                if li in out_last:
                    y0, y1 = lio[out_last[li]][2], lio[li][2] + lio[li][3]
                    done = torch.cuda.Event()
                    done.record(stream)
                    cs_out.wait_event(done)
                    with torch.cuda.stream(cs_out):
                        YH[y0:y1].copy_(Y[y0:y1], non_blocking=True)
            join = torch.cuda.Event()
            join.record(cs_out)
            stream.wait_event(join)

        def e2e_step():  # noqa: F811 (the pipelined form for the chain)
            g_e2e.replay()

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
    ems = max_over_ranks(f0.elapsed_time(f1), "cuda")

    peaks = {}
    try:
        peaks = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))
    except (OSError, ValueError):
        pass
    hbm = peaks.get("hbm_gbs")
    peak_src = "measured" if hbm else "fallback"
    hbm = hbm or 6650.0
    result = {
        "metric": METRIC, "value": round(gbs, 2), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_step, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": dtype_of(args.workload),
        "data": "synthetic (seeded, kqgen)",
        "tok_per_s": round(tok_s, 3), "frac_of_hbm_peak": round(gbs / world / hbm, 4),
        "config": workload_config(args.workload, world),
        "e2e": {"value": round(job_rate(wl.weight_bytes, args.steps, world, ems) / 1e9, 2), "unit": "GB/s",
                "tok_per_s": round(job_rate(k, args.steps, world, ems), 3),
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "clocks": clk.summary(),
        "gpu_launches": (wl.launches_per_step if getattr(wl, "use_steps", False) else len(wl.launches)) * args.steps,
    }
    if per_kind:
        dom = max(per_kind, key=lambda n: per_kind[n]["share"])
        dk = per_kind[dom]
        kname = ("mma_kernel (tensor cores)" if k >= 2 else
                 "steps_kernel (multi-step launch)" if getattr(wl, "use_steps", False) else
                 "gemv_kernel (routed segments)" if isinstance(wl, MoE) else "gemv1_kernel")
        rd = read_roofline(torch, kq)
        rpk = max(rd.values())
        result["roofline"] = {"bound": "hbm", "kernel": f"{kname} {dk['fmt']} {dom} {dk['N']}x{dk['K']}",
                              "achieved": dk["gbs"], "peak": hbm, "peak_source": f"{peak_src} copy (read+write)",
                              "unit": "GB/s", "frac": round(dk["gbs"] / hbm, 4),
                              "read_peak": rd, "frac_of_read_peak": round(dk["gbs"] / rpk, 4),
                              "frac_of_nominal_8tbs": round(dk["gbs"] / 8000.0, 4),
                              "traffic": measured_traffic(dk["fmt"], dk["N"], dk["K"], k),
                              "algorithmic_bytes": dk["bytes"]}
        result["frac_of_read_peak"] = round(gbs / world / rpk, 4)
        result["kernels"] = per_kind
    if isinstance(wl, (Streamed, MoEStreamed)):
        pk = h2d_peak_gbs(torch)
        h2d = job_rate(wl.streamed_bytes, args.steps, world, ms) / 1e9 / world
        result["roofline"] = {"bound": "pcie_h2d",
                              "kernel": "H2D copies of the routed experts" if isinstance(wl, MoEStreamed)
                              else "H2D copies of the layer ring",
                              "achieved": round(h2d, 2), "peak": round(pk, 2),
                              "peak_source": "measured here (512 MiB pinned copy)", "unit": "GB/s",
                              "frac": round(h2d / pk, 4), "traffic": None,
                              "streamed_bytes_per_step": wl.streamed_bytes, "resident_layers": wl.n_resident}
        result["gpu_launches"] = len(wl.launches) * args.steps
    return result


def cpu_baseline(args, budget_s=15.0, single_s=5.0):
    """The oracle as it stands, on a bounded sample of the workload: the
    first rows of each matrix of the leading layers, timed on all host cores
    (OpenMP over rows) and, on a smaller share of the same sample, on one
    core.  For the 70B-shaped chains the sample is at most the first 4
    layers and tok/s is extrapolated from the sample's byte rate to the
    whole chain's bytes per token."""
    import kqgen
    import oracle

    spec, _ = workload_spec(args.workload)
    if spec is None:
        spec = [[("moe_gate_up", "q4_k", 2 * MOE30B["ffn"], MOE30B["hidden"], 0),
                 ("moe_down", "q4_k", MOE30B["hidden"], MOE30B["ffn"], 1)]] * MOE30B["layers"]
    per_token = workload_config(args.workload, 1)["weight_bytes_per_step"]
    max_layers = 4 if CHAIN_BASE.get(args.workload) == "llama70b" else len(spec)
    cores = len(os.sched_getaffinity(0))
    fused = args.workload.startswith("llama8b_layer_fused")

    def run(nthreads, budget):
        done_bytes, t_total, rows_done, li = 0, 0.0, 0, 0
        t_start = time.time()
        while time.time() - t_start < budget and li < min(len(spec), max_layers):
            for mi, (name, fmt, N, K, slot) in enumerate(spec[li]):
                nrows = min(N, 512)
                W = kqgen.matrix(fmt, kqgen.tensor_seed(SEED, li, mi), nrows, K)
                x = kqgen.normal_f32(kqgen.tensor_seed(SEED ^ 0x5A5A, li, 0 if slot is None else slot), K)
                t0 = time.perf_counter()
                if fused and name != "o":
                    # the fused forms: RMSNorm (unit weights) before qkv and
                    # gate|up, the SiLU-gated product of a [g; u] input before down
                    if name == "down":
                        gu = kqgen.normal_f32(kqgen.tensor_seed(SEED ^ 0x5A5A, li, 3), 2 * K)
                        oracle.gemv_fused(fmt, W, nrows, K, gu, "swiglu", nthreads=nthreads)
                    else:
                        oracle.gemv_fused(fmt, W, nrows, K, x, "rmsnorm", np.ones(K, np.float32), 1e-5,
                                          nthreads=nthreads)
                else:
                    oracle.gemv(fmt, W, nrows, K, x, nthreads=nthreads)
                t_total += time.perf_counter() - t0
                done_bytes += nrows * row_bytes(fmt, K)
                rows_done += nrows
            li += 1
        return done_bytes / t_total / 1e9, li, rows_done, done_bytes

    gbs, li, rows_done, done_bytes = run(cores, budget_s)
    gbs1, li1, rows1, bytes1 = run(1, single_s)
    extrap = (f"; tok/s extrapolated from the sample's rate to the whole chain's {per_token / 1e9:.2f} GB per token"
              if max_layers < len(spec) else "")
    return {"value": round(gbs, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
            "tok_per_s": round(gbs * 1e9 / per_token, 6),
            "sample": f"first <=512 rows of each matrix of {li} layer(s) ({rows_done} rows, "
                      f"{done_bytes / 1e6:.1f} MB of weights), fp64 oracle, OpenMP over rows{extrap}",
            "single_thread": {"value": round(gbs1, 4), "unit": "GB/s", "cores": 1,
                              "tok_per_s": round(gbs1 * 1e9 / per_token, 6),
                              "sample": f"first <=512 rows of each matrix of {li1} layer(s) ({rows1} rows, "
                                        f"{bytes1 / 1e6:.1f} MB), one thread"}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="llama8b_chain", choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="kq", choices=["kq", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.steps is None:
        args.steps = {"llama70b_stream": 3, "llama70b_stream_20gb": 5, "llama70b_resident": 50,
                      "llama70b_resident_steps": 50}.get(args.workload, 300)
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))

    if args.impl == "reference":
        if rank != 0:
            return
        cb = cpu_baseline(args, budget_s=min(60.0, max(5.0, 1.0 * args.steps)))
        line = {"metric": METRIC, "value": cb["value"], "unit": "GB/s", "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "f64", "data": "synthetic (seeded, kqgen)", "impl": "reference",
                "config": workload_config(args.workload, world),
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
