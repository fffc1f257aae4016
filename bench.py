#!/usr/bin/env python
"""Benchmark of the MoonEP balanced expert-parallel hot path on B200.

One step = one MoE layer's pass of the whole hot path over a fresh batch of
router output: plan -> (training: prefetch of replica weights) -> zero-copy
dispatch -> identity expert -> combine, and in training mode combine-backward ->
dispatch-backward -> reduce_grad of replica expert gradients.
Inputs are synthetic and seeded (Zipf-popular experts, Gumbel-top-k picks,
softmax gates, N(0,1) bf16 rows; see moonep_inputs).

Metric (headline): dispatch+combine HBM GB/s = algorithmic bytes of the two
kernels / their CUDA-event time, plus plan µs per layer.  ms_per_step comes from
K steps with events only around them (kernels overlap their launch gaps as in
use); the per-kernel times, the metric and the roofline from a second pass of
K steps with an event after every kernel; `b2b_ms` per data kernel from ten
launches in a row between two events (no event between launches).  Training
workloads also report `reduce_grad_f32`: the same fold over fp32 gradient buffers
on the step's plan (not part of the step), timed the same two ways.
Default workload: R=8 ranks, E=256 experts, K=8, S=4096 tokens/rank, H=7168,
maxvio 0.2, replica budget 32 (training).  The default run then adds, on the
same line: `sweep` — the forward layer (plan + dispatch + combine) of the same
shape at maxvio 0.2, 1, 2, 5, 10, 20 over two seeds, with the flatness of the
layer time; `decode` — the 64-rank inference workload at maxvio 1 and 20; and
`cpu_baseline` — the CPU oracle on a bounded sample, single-threaded and on
every host core.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--maxvio M]
    python bench.py --sweep            # maxvio 0.2..20 x 5 seeds, one JSON line per maxvio
    python bench.py --impl reference   # the CPU oracle on a bounded sample, same metric

With N > 1 (torchrun), every rank runs an independent replica of the layer on
its own GPU (weak scaling, no data-path collective); rank 0 prints one line
with the whole-job value (bytes of all ranks / the slowest rank's time).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from moonep_inputs import (MODE_TRAIN, WORKLOADS, make_dout, make_gates, make_routing,  # noqa: E402
                           make_x, normal_bf16)

METRIC = "dispatch+combine HBM GB/s (% of peak) and plan µs/layer vs maxvio, 1×B200"
DEFAULT_WORKLOAD = "ep8_e256_k8_s4096_h7168"
DECODE_WORKLOAD = "ep64_e256_k8_s128_h7168_decode"
SWEEP_MAXVIO = (0.2, 1.0, 2.0, 5.0, 10.0, 20.0)
FALLBACK_HBM_GBS = 6650.0
NOMINAL_HBM_GBS = 8000.0


# ------------------------------------------------------------------ bytes ---
def algorithmic_bytes(R, S, K, H, n_local=0, n_rep_exp=0, P=0):
    """Bytes each kernel must move (bf16 = 2 B), per launch; re-reads and padding excluded."""
    T = R * S
    RSK = T * K
    return {
        "plan": RSK * 4 * 2,  # router ids in, slot map out
        "dispatch": T * H * 2 + RSK * H * 2 + RSK * 4,
        "combine": RSK * H * 2 + T * H * 2 + RSK * 8,
        "combine_bwd": T * H * 2 + 2 * RSK * H * 2 + RSK * 12,
        "reduce_grad": n_local * P * 2 + n_rep_exp * P * 2 * 2,
        "prefetch": n_rep_exp * P * 2 + n_local * P * 2,  # home weights read once, replicas written
        "dispatch_bwd": RSK * H * 2 + T * H * 2 + RSK * 4,
    }


def hbm_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            v = float(json.load(f)["hbm_gbs"])
        return v, "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def ncu_traffic(workload, maxvio, seed):
    """Per-kernel DRAM bytes per launch from the committed ncu summary, if it was taken on
    this workload (name, maxvio, seed) and neither the kernel's source nor the shared
    header has changed since."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "ncu_traffic.txt")
    out = {}
    try:
        lines = open(path).read().splitlines()
    except OSError:
        return out
    src_hash = {}
    for f in ("plan.cu", "data.cu", "moonep_internal.cuh"):
        try:
            with open(os.path.join(ROOT, "token_dispatch_moonep_b200", "csrc", f), "rb") as fh:
                src_hash[f] = hashlib.sha256(fh.read()).hexdigest()[:16]
        except OSError:
            pass
    for ln in lines:
        if ln.startswith("#") or not ln.strip():
            continue
        parts = dict(kv.split("=", 1) for kv in ln.split())
        same_case = (parts.get("workload") == workload and parts.get("seed") == str(seed)
                     and abs(float(parts.get("maxvio", "nan")) - maxvio) < 1e-9)
        same_src = (src_hash.get(parts.get("source")) == parts.get("sha") and
                    parts.get("header_sha", src_hash.get("moonep_internal.cuh"))
                    == src_hash.get("moonep_internal.cuh"))
        if same_case and same_src:
            out[parts["kernel"]] = float(parts["bytes_per_launch"])
    return out


# ----------------------------------------------------------------- clocks ---
class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 100 ms during the timed region."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index=0):
        import torch
        self.proc = None
        try:
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            sel = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", sel, f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            return None
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in out.splitlines():
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 8:
                continue
            try:
                sm.append(float(f[0]))
                mx.append(float(f[1]))
            except ValueError:
                continue
            for n, v in zip(names, f[4:8]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "samples": len(sm),
                "reasons": sorted(reasons)}


def merge_clocks(parts):
    """One clocks record over several sampled regions (median of the medians, all reasons)."""
    parts = [c for c in parts if c]
    if not parts:
        return None
    return {"sm_mhz": statistics.median(c["sm_mhz"] for c in parts),
            "sm_min_mhz": min(c["sm_mhz"] for c in parts),
            "sm_max_mhz": max(c["sm_max_mhz"] for c in parts),
            "samples": sum(c["samples"] for c in parts),
            "reasons": sorted(set().union(*[set(c["reasons"]) for c in parts]))}


# ------------------------------------------------------------- GPU layer ---
class Layer:
    """Device buffers and the per-step call sequence of one MoE layer."""

    def __init__(self, w, maxvio, seed, device, with_backward=None, host_inputs=True):
        import torch
        import token_dispatch_moonep_b200 as me
        self.me, self.torch, self.w = me, torch, w
        self.dev = device
        self.train = (w.mode == MODE_TRAIN) if with_backward is None else with_backward
        R, E, K, S, H = w.R, w.E, w.K, w.S, w.H
        self.cfg = me.Config.of(w)
        self.NvS = me.moonep_nvs(self.cfg)
        T = R * S
        pin = torch.cuda.is_available()
        self.pin = pin
        if host_inputs:
            self.h_x = torch.from_numpy(make_x(R, S, H, seed).reshape(-1).view(np.int16))
            self.h_dout = (torch.from_numpy(make_dout(R, S, H, seed).reshape(-1).view(np.int16))
                           if self.train else None)
        else:
            g = torch.Generator(device=device).manual_seed(seed)
            self.h_x = torch.randn(T * H, generator=g, device=device).to(torch.bfloat16).view(torch.int16).cpu()
            self.h_dout = (torch.randn(T * H, generator=g, device=device).to(torch.bfloat16)
                           .view(torch.int16).cpu() if self.train else None)
        if pin:
            self.h_x = self.h_x.pin_memory()
            if self.h_dout is not None:
                self.h_dout = self.h_dout.pin_memory()
        self.idx = torch.empty(T * K, dtype=torch.int32, device=device)
        self.gates = torch.empty(T * K, dtype=torch.float32, device=device)
        self.set_routing(maxvio, seed)
        self.x = self.h_x.to(device)
        self.recv = torch.empty(R * self.NvS * H, dtype=torch.int16, device=device)
        self.out = torch.empty(T * H, dtype=torch.int16, device=device)
        self.arena, self.ws, self.status = me.alloc_plan(self.cfg, device)
        if self.train:
            self.P = w.P or 2048 * H
            self.dout = self.h_dout.to(device)
            self.dy = torch.empty_like(self.recv)
            self.dg = torch.empty(T * K, dtype=torch.float32, device=device)
            g = torch.Generator(device=device).manual_seed(seed + 1)
            self.rep = torch.empty(R * w.budget * self.P, dtype=torch.bfloat16, device=device)
            self.home = torch.empty(E * self.P, dtype=torch.bfloat16, device=device)
            for buf in (self.rep, self.home):  # N(0,1) in chunks to bound fp32 temporaries
                n = buf.numel()
                step = 1 << 28
                for i in range(0, n, step):
                    buf[i:i + step].copy_(torch.randn(min(step, n - i), generator=g, device=device))
            self.dx = torch.empty(T * H, dtype=torch.int16, device=device)
            self.weights = torch.empty(E * self.P, dtype=torch.bfloat16, device=device)
            self.rep_w = torch.empty(R * w.budget * self.P, dtype=torch.bfloat16, device=device)
            self.weights.copy_(self.home)  # any bf16 values: the copy moves bits
            self.h_out = torch.empty(T * H, dtype=torch.int16).pin_memory() if pin else None
            self.h_dg = torch.empty(T * K, dtype=torch.float32).pin_memory() if pin else None
        else:
            self.P = 0
            self.h_out = torch.empty(T * H, dtype=torch.int16).pin_memory() if pin else None
        self.n_local = self.n_rep_exp = self.n_piece = self.n_remote = 0
        self.e2e_bufs = None

    def set_routing(self, maxvio, seed):
        """New router output (tuned to `maxvio`) and gates in the same device buffers."""
        torch, w = self.torch, self.w
        idx, self.alpha, self.maxvio = make_routing(w.R, w.E, w.K, w.S, maxvio, seed)
        gates = make_gates(w.R, w.S, w.K, seed)
        self.h_idx = torch.from_numpy(idx.ravel().copy())
        self.h_gates = torch.from_numpy(gates.ravel().copy())
        if self.pin:
            self.h_idx = self.h_idx.pin_memory()
            self.h_gates = self.h_gates.pin_memory()
        self.idx.copy_(self.h_idx)
        self.gates.copy_(self.h_gates)
        self.torch.cuda.synchronize()

    def alloc_e2e(self):
        """Second set of input and output buffers so copies of one step overlap another."""
        torch = self.torch
        if self.e2e_bufs is None:
            second = dict(idx=torch.empty_like(self.idx), gates=torch.empty_like(self.gates),
                          x=torch.empty_like(self.x), out=torch.empty_like(self.out))
            first = dict(idx=self.idx, gates=self.gates, x=self.x, out=self.out)
            h_out = [self.h_out, torch.empty_like(self.h_out).pin_memory()]
            if self.train:
                second.update(dout=torch.empty_like(self.dout), dg=torch.empty_like(self.dg))
                first.update(dout=self.dout, dg=self.dg)
                h_dg = [self.h_dg, torch.empty_like(self.h_dg).pin_memory()]
            else:
                h_dg = [None, None]
            self.e2e_bufs = ([first, second], h_out, h_dg)
        return self.e2e_bufs

    def ops(self, buf=None, forward_only=False):
        """The step's ABI calls; `buf` selects an input/output buffer set (default: the
        first); `forward_only` keeps plan, dispatch and combine."""
        me, c = self.me, self.cfg
        train = self.train and not forward_only
        b = buf or dict(idx=self.idx, gates=self.gates, x=self.x, out=self.out,
                        dout=getattr(self, "dout", None), dg=getattr(self, "dg", None))
        seq = [("plan", lambda: me.moonep_plan(c, b["idx"], self.arena, self.ws, self.status))]
        if train:
            seq += [("prefetch", lambda: me.moonep_prefetch_weight(c, self.arena, self.weights, self.rep_w,
                                                                   self.P, self.status))]
        seq += [("dispatch", lambda: me.moonep_dispatch(c, self.arena, b["x"], self.recv, self.status)),
               ("combine", lambda: me.moonep_combine(c, self.arena, self.recv, b["gates"], b["out"],
                                                     self.status))]
        if train:
            seq += [("combine_bwd", lambda: me.moonep_combine_backward(
                        c, self.arena, b["dout"], self.recv, b["gates"], self.dy, b["dg"],
                        self.status)),
                    ("dispatch_bwd", lambda: me.moonep_dispatch_backward(c, self.arena, self.dy, self.dx,
                                                                         self.status)),
                    ("reduce_grad", lambda: me.moonep_reduce_grad(c, self.arena, self.rep, self.home,
                                                                  self.P, self.status))]
        return seq

    def read_plan_stats(self):
        v = self.me.moonep_plan_view(self.cfg, self.arena)
        sc = v["scalars"].cpu().numpy()
        self.n_local, self.n_rep_exp = int(sc[2]), int(sc[3])
        self.n_piece, self.n_remote = int(sc[0]), int(sc[1])

    def bytes(self, forward_only=False):
        w = self.w
        b = algorithmic_bytes(w.R, w.S, w.K, w.H, self.n_local, self.n_rep_exp, self.P)
        if not self.train or forward_only:
            for k in ("combine_bwd", "reduce_grad", "prefetch", "dispatch_bwd"):
                b.pop(k)
        return b


def time_steps(layer, steps, warmup, barrier=None, ops=None):
    """Warm up, then time `steps` steps twice on the current stream.

    Pass 1 is the timed region of the result line: events only before the first
    and after the last step, so consecutive kernels overlap their launch gaps
    (every data kernel uses programmatic dependent launch) exactly as they do
    for a caller.  Pass 2 repeats the steps with an event after every kernel for
    the per-kernel breakdown; an event between two kernels ends that overlap,
    so per-kernel times carry a few microseconds more than pass 1 accounts for."""
    torch = layer.torch
    ops = ops or layer.ops()
    layer.status.zero_()
    for _ in range(warmup):
        for _, fn in ops:
            fn()
    torch.cuda.synchronize()
    layer.read_plan_stats()
    stream = torch.cuda.current_stream()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(ops) + 1)] for _ in range(steps)]
    if barrier:
        barrier()
    torch.cuda.synchronize()
    sampler = ClockSampler(torch.cuda.current_device())
    time.sleep(0.25)  # let the sampler start before the timed region
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for s in range(steps):
        for _, fn in ops:
            fn()
    t1.record(stream)
    torch.cuda.synchronize()
    if barrier:
        barrier()
    for _, fn in ops:  # one untimed step: the first launch after the host sync starts cold
        fn()
    for s in range(steps):
        ev[s][0].record(stream)
        for i, (_, fn) in enumerate(ops):
            fn()
            ev[s][i + 1].record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    if barrier:
        barrier()
    total_ms = t0.elapsed_time(t1)
    per = {name: [ev[s][i].elapsed_time(ev[s][i + 1]) for s in range(steps)]
           for i, (name, _) in enumerate(ops)}
    st = int(layer.status.item())
    return total_ms, per, clocks, st


def time_back_to_back(layer, n=10, ops=None):
    """Each data kernel launched n times in a row between two events (after two untimed
    launches): its average launch duration without an event between launches, which
    otherwise adds a few microseconds to every launch.  The plan is left out: its
    latency inside the step is what counts."""
    torch = layer.torch
    out = {}
    for name, fn in (ops or layer.ops()):
        if name == "plan":
            continue
        fn()
        fn()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(n):
            fn()
        e1.record()
        torch.cuda.synchronize()
        out[name] = e0.elapsed_time(e1) / n
    return out


def time_reduce_grad_f32(layer, n=10):
    """reduce_grad over fp32 gradient buffers (moonep_reduce_grad_f32; not one of the
    step's kernels: the step folds bf16 gradients) on the step's plan and row length:
    its launch time with events around each launch and launched n times back to back,
    against its algorithmic bytes (the bf16 fold's, at 4 bytes a value)."""
    torch, me, w = layer.torch, layer.me, layer.w
    g = torch.Generator(device=layer.dev).manual_seed(7)
    rep = torch.randn(w.R * w.budget * layer.P, generator=g, device=layer.dev)
    home = torch.randn(w.E * layer.P, generator=g, device=layer.dev)
    fn = lambda: me.moonep_reduce_grad_f32(layer.cfg, layer.arena, rep, home, layer.P, layer.status)
    fn()
    fn()
    ev = lambda: torch.cuda.Event(enable_timing=True)
    each = []
    for _ in range(n):
        e0, e1 = ev(), ev()
        e0.record()
        fn()
        e1.record()
        each.append((e0, e1))
    e0, e1 = ev(), ev()
    e0.record()
    for _ in range(n):
        fn()
    e1.record()
    torch.cuda.synchronize()
    ms = sum(a.elapsed_time(c) for a, c in each) / n
    b2b = e0.elapsed_time(e1) / n
    nbytes = 2 * layer.bytes()["reduce_grad"]
    del rep, home
    torch.cuda.empty_cache()
    return {"ms": ms, "b2b_ms": b2b, "bytes": nbytes, "GBs": nbytes / (ms * 1e-3) / 1e9,
            "b2b_GBs": nbytes / (b2b * 1e-3) / 1e9}


def host_cost(layer, n=500):
    """Host time of one enqueue through the C ABI (ctypes call with pointers already
    marshalled; the GPU work queues up behind), in µs per call: the library's argument
    checks, its cached launch facts and the launch itself."""
    import ctypes
    torch, me, c = layer.torch, layer.me, layer.cfg
    lib = me._lib
    s = torch.cuda.current_stream().cuda_stream
    cp = ctypes.byref(c)
    calls = {
        "plan": lambda: lib.moonep_plan(cp, layer.idx.data_ptr(), layer.arena.data_ptr(),
                                        layer.ws.data_ptr(), layer.status.data_ptr(), s),
        "dispatch": lambda: lib.moonep_dispatch(cp, layer.arena.data_ptr(), layer.x.data_ptr(),
                                                layer.recv.data_ptr(), layer.status.data_ptr(), s),
    }
    out = {}
    for name, fn in calls.items():
        torch.cuda.synchronize()
        fn()
        t0 = time.perf_counter()
        for _ in range(n):
            fn()
        out[name] = (time.perf_counter() - t0) / n * 1e6
        torch.cuda.synchronize()
    return out


def time_e2e(layer, steps):
    """The same steps through the public API from host memory, pipelined as a user would:
    step s+1's inputs are copied in from pinned host memory (H2D stream) and step s-1's
    results read back (D2H stream) while step s computes.  Two buffer sets."""
    torch = layer.torch
    bufs, h_out, h_dg = layer.alloc_e2e()
    comp = torch.cuda.current_stream()
    h2d = torch.cuda.Stream()
    d2h = torch.cuda.Stream()
    ev = lambda: torch.cuda.Event(enable_timing=False)
    n = steps + 2
    in_ready = [ev() for _ in range(n)]
    comp_done = [ev() for _ in range(n)]
    out_done = [ev() for _ in range(n)]
    ops = [layer.ops(bufs[0]), layer.ops(bufs[1])]

    def copy_in(s):
        b = bufs[s % 2]
        with torch.cuda.stream(h2d):
            if s >= 2:
                h2d.wait_event(comp_done[s - 2])  # the buffer set is free again
            b["idx"].copy_(layer.h_idx, non_blocking=True)
            b["gates"].copy_(layer.h_gates, non_blocking=True)
            b["x"].copy_(layer.h_x, non_blocking=True)
            if layer.train:
                b["dout"].copy_(layer.h_dout, non_blocking=True)
            in_ready[s].record(h2d)

    def run(s, start=None):
        b = bufs[s % 2]
        comp.wait_event(in_ready[s])
        if s >= 2:
            comp.wait_event(out_done[s - 2])  # its outputs were read back
        for _, fn in ops[s % 2]:
            fn()
        comp_done[s].record(comp)
        with torch.cuda.stream(d2h):
            d2h.wait_event(comp_done[s])
            h_out[s % 2].copy_(b["out"], non_blocking=True)
            if layer.train:
                h_dg[s % 2].copy_(b["dg"], non_blocking=True)
            out_done[s].record(d2h)

    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(h2d)
    copy_in(0)
    for s in range(steps):
        if s + 1 < steps:
            copy_in(s + 1)
        run(s)
    t1.record(d2h)
    torch.cuda.synchronize()
    ms = t0.elapsed_time(t1)
    h2d_b = (layer.h_idx.numel() * 4 + layer.h_gates.numel() * 4 + layer.h_x.numel() * 2 +
             (layer.h_dout.numel() * 2 if layer.train else 0))
    d2h_b = layer.h_out.numel() * 2 + (layer.h_dg.numel() * 4 if layer.train else 0)
    return ms, h2d_b, d2h_b


def max_over_ranks(pg, values, device):
    """Element-wise max of per-rank timings (identity for one process)."""
    if pg is None:
        return list(values)
    import torch
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return t.tolist()


def whole_job_gbs(bytes_per_rank, world, ms):
    """Units all ranks processed divided by the slowest rank's time, in GB/s."""
    return bytes_per_rank * world / (ms * 1e-3) / 1e9


def workload_config(w, maxvio, alpha, world, scaled=False):
    """The `config` object of the result line (shared by both arms)."""
    NvS = w.S * w.K + (w.align - 1) * min(w.E, w.S * w.K)
    train = w.mode == MODE_TRAIN
    return {"workload": w.name + (f"/S{w.S}" if scaled else ""),
            "R": w.R, "E": w.E, "K": w.K, "S": w.S, "H": w.H, "budget": w.budget,
            "mode": "train" if train else "infer",
            "maxvio": round(maxvio, 4), "zipf_alpha": round(alpha, 4),
            "step": ("plan+prefetch+dispatch+combine+combine_bwd+dispatch_bwd+reduce_grad"
                     if train else "plan+dispatch+combine"),
            "grad_elems_per_expert": (w.P or 2048 * w.H) if train else 0,
            "l2": "inputs larger than L2 (x %.0f MB, dispatch buffer %.0f MB); no flush"
                  % (w.R * w.S * w.H * 2 / 1e6, w.R * NvS * w.H * 2 / 1e6),
            "parallelism": f"{world} independent replica(s), one per GPU"}


# ------------------------------------------------------ sweep and decode ---
def forward_pass(layer, steps, warmup):
    """Plan + dispatch + combine of the layer's current routing: per-kernel medians and
    the overlapped layer time (pass 1 of time_steps)."""
    ops = layer.ops(forward_only=True)
    total_ms, per, clocks, st = time_steps(layer, steps, warmup, ops=ops)
    b = layer.bytes(forward_only=True)
    med = {k: statistics.median(v) for k, v in per.items()}
    return {"maxvio": round(layer.maxvio, 4), "alpha": round(layer.alpha, 4),
            "plan_us": med["plan"] * 1e3,
            "dispatch_GBs": b["dispatch"] / med["dispatch"] / 1e6,
            "combine_GBs": b["combine"] / med["combine"] / 1e6,
            "layer_us": 1e3 * total_ms / steps,
            "layer_us_kernel_events": 1e3 * (med["plan"] + med["dispatch"] + med["combine"]),
            "pieces": layer.n_piece, "remote": layer.n_remote, "status": st}, clocks


def compact_sweep(layer, seeds, steps, warmup, targets=SWEEP_MAXVIO):
    """The forward layer of `layer`'s shape across router imbalance, reusing its buffers."""
    peak, _ = hbm_peak()
    rows, clocks = [], []
    for mv in targets:
        per_seed = []
        for seed in seeds:
            layer.set_routing(mv, seed)
            r, c = forward_pass(layer, steps, warmup)
            r["seed"] = seed
            per_seed.append(r)
            clocks.append(c)
        row = {"target_maxvio": mv}
        for k in ("maxvio", "plan_us", "dispatch_GBs", "combine_GBs", "layer_us",
                  "layer_us_kernel_events", "pieces"):
            row[k] = statistics.mean(r[k] for r in per_seed)
        row["status"] = max(r["status"] for r in per_seed)
        row["seeds"] = per_seed
        rows.append(row)
    lay = [r["layer_us"] for r in rows]
    plan = [r["plan_us"] for r in rows]
    return {"workload": layer.w.name, "seeds": list(seeds), "steps": steps,
            "layer": "plan+dispatch+combine, overlapped launches (events only around the steps)",
            "flatness": max(lay) / min(lay), "plan_flatness": max(plan) / min(plan),
            "peak_GBs": peak, "rows": rows, "clocks": merge_clocks(clocks)}


def fused_pass(layer, steps, warmup):
    """The same forward layer as one launch (moonep_fused_forward: plan, dispatch and the
    identity expert's combine): overlapped layer time and per-call event time."""
    me, c = layer.me, layer.cfg
    ops = [("fused", lambda: me.moonep_fused_forward(c, layer.idx, layer.gates, layer.x, layer.arena,
                                                     layer.ws, layer.recv, layer.out, layer.status))]
    total_ms, per, clocks, st = time_steps(layer, steps, warmup, ops=ops)
    return {"fused_layer_us": 1e3 * total_ms / steps,
            "fused_layer_us_kernel_events": 1e3 * statistics.median(per["fused"]),
            "fused_status": st}, clocks


def graph_pass(layer, layers=10, replays=4):
    """The forward layer (plan, dispatch, combine) as a serving loop would run it: `layers`
    layers captured in one CUDA graph (the plan's launch epoch advances on every replay),
    replayed `replays` times between two events; (µs per layer, device status)."""
    torch = layer.torch
    ops = layer.ops(forward_only=True)
    layer.status.zero_()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        for _, fn in ops:  # first calls (cached launch facts) before the capture
            fn()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        for _ in range(layers):
            for _, fn in ops:
                fn()
    with torch.cuda.stream(s):
        g.replay()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(s)
        for _ in range(replays):
            g.replay()
        e1.record(s)
    torch.cuda.synchronize()
    us = e0.elapsed_time(e1) * 1e3 / (layers * replays)
    del g
    return us, int(layer.status.item())


def decode_runs(device, steps, warmup, maxvios=(1.0, 20.0), seed=0):
    """The 64-rank inference workload: plan + dispatch + combine µs per maxvio, as three
    calls, as the same three calls replayed from a CUDA graph of ten layers, and as the
    one-launch fused layer."""
    w = WORKLOADS[DECODE_WORKLOAD]
    layer = Layer(w, maxvios[0], seed, device, with_backward=False, host_inputs=False)
    out, clocks = [], []
    for mv in maxvios:
        layer.set_routing(mv, seed)
        r, c = forward_pass(layer, steps, warmup)
        r["graph_layer_us"], r["graph_status"] = graph_pass(layer)
        fr, fc = fused_pass(layer, steps, warmup)
        r.update(fr)
        out.append(r)
        clocks += [c, fc]
    b = layer.bytes(forward_only=True)
    res = {"workload": w.name, "seed": seed, "steps": steps,
           "bytes_dispatch_combine": b["dispatch"] + b["combine"],
           "rows": out, "clocks": merge_clocks(clocks)}
    del layer
    return res


# ------------------------------------------------------------ CPU oracle ---
def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def _run_threads(fn, parts):
    """fn(part) on one thread per part (the oracle's C calls release the GIL)."""
    if len(parts) == 1:
        fn(parts[0])
        return
    ths = [threading.Thread(target=fn, args=(p,)) for p in parts]
    for t in ths:
        t.start()
    for t in ths:
        t.join()


def _time_until(fn, min_s):
    """Repeat fn until at least min_s seconds have passed; (reps, seconds)."""
    reps, t0 = 0, time.perf_counter()
    while True:
        fn()
        reps += 1
        el = time.perf_counter() - t0
        if el >= min_s:
            return reps, el


class OracleSample:
    """The unchanged CPU oracle on a bounded sample of a workload: the first `s` tokens of
    every rank of the same seeded routing, planned as one layer of S = s tokens, and
    expert-gradient / weight rows cut to their first `p` elements."""

    def __init__(self, w, maxvio, seed, s, p=1 << 18):
        import oracle
        self.o = oracle
        R, E, K, H, B = w.R, w.E, w.K, w.H, w.budget
        idx, _, _ = make_routing(R, E, K, w.S, maxvio, seed)
        self.idx = np.ascontiguousarray(idx[:, :s, :])
        self.gates = np.ascontiguousarray(make_gates(R, w.S, K, seed)[:, :s, :]).reshape(R * s, K)
        self.x = make_x(R, s, H, seed).reshape(R * s, H)
        self.dout = make_dout(R, s, H, seed).reshape(R * s, H)
        self.cfg = oracle.Config(R=R, E=E, K=K, S=s, H=H, budget=w.budget, mode=w.mode)
        self.R, self.E, self.K, self.H, self.B, self.s, self.P = R, E, K, H, B, s, p
        self.train = w.mode == MODE_TRAIN
        st, self.t = oracle.plan(self.cfg, self.idx)
        self.slot_of = self.t["slot_of"]
        self.NvS = int(self.t["nvs"][0])
        self.recv = np.zeros((R * self.NvS, H), np.uint16)
        self.out = np.zeros((R * s, H), np.uint16)
        self.dy = np.zeros((R * self.NvS, H), np.uint16)
        local = self.t["piece_wslot"] >= 0
        self.n_local = int(local.sum())
        self.rep_experts = np.unique(self.t["piece_expert"][local])
        if self.train:
            # N(0,1) rows (no subnormal values, which would slow the host arithmetic down);
            # only the slots of local pieces are ever read
            self.home = normal_bf16((E, p), seed, stream=21)
            self.rep = np.zeros((R, max(B, 1), p), np.uint16)
            li = np.nonzero(local)[0]
            rows = normal_bf16((max(len(li), 1), p), seed, stream=22)
            for j, i in enumerate(li):
                self.rep[self.t["piece_rank"][i], self.t["piece_wslot"][i]] = rows[j]
            self.weights = self.home.copy()
            self.rep_w = np.zeros_like(self.rep)

    def bytes(self):
        return algorithmic_bytes(self.R, self.s, self.K, self.H, self.n_local,
                                 len(self.rep_experts), self.P)

    def kernels(self):
        """name -> callable(n_threads) running that step of the oracle once."""
        o, c, K, H = self.o, self.cfg, self.K, self.H
        T = self.R * self.s

        def token_parts(n):
            return [p for p in np.array_split(np.arange(T, dtype=np.int64), n) if p.size]

        def dispatch(n):
            def part(tk):
                t0, t1 = int(tk[0]), int(tk[-1]) + 1
                sub = o.Config(R=1, E=c.E, K=K, S=t1 - t0, H=H, budget=c.budget, mode=c.mode)
                o.dispatch(sub, self.slot_of[t0 * K:t1 * K], self.x[t0:t1], self.recv)
            _run_threads(part, token_parts(n))

        def combine(n):
            _run_threads(lambda tk: o.combine(c, self.slot_of, self.recv, self.gates, tk),
                         token_parts(n))

        def combine_bwd(n):
            _run_threads(lambda tk: o.combine_backward(c, self.slot_of, self.dout, self.recv,
                                                       self.gates, tk), token_parts(n))

        def dispatch_bwd(n):
            _run_threads(lambda tk: o.dispatch_backward(c, self.slot_of, self.dy, tk),
                         token_parts(n))

        def expert_parts(n):
            groups = [g for g in np.array_split(self.rep_experts, n) if g.size]
            out = []
            for g in groups:
                m = np.isin(self.t["piece_expert"], g)
                out.append({k: self.t[k][m] for k in ("piece_expert", "piece_rank", "piece_wslot")})
            return out or [{k: self.t[k][:0] for k in ("piece_expert", "piece_rank",
                                                        "piece_wslot")}]

        def reduce_grad(n):
            _run_threads(lambda tb: o.reduce_grad(c, tb, self.rep, self.home, inplace=True),
                         expert_parts(n))

        def prefetch(n):
            _run_threads(lambda tb: o.prefetch_weight(c, tb, self.weights, self.rep_w, inplace=True),
                         expert_parts(n))

        ks = {"dispatch": dispatch, "combine": combine}
        if self.train:
            ks.update(prefetch=prefetch, combine_bwd=combine_bwd, dispatch_bwd=dispatch_bwd,
                      reduce_grad=reduce_grad)
        return ks


def oracle_baseline(w, maxvio, seed, s_sample, min_s=1.0):
    """The CPU oracle, as it stands, on a bounded sample: the plan single-threaded (its
    algorithm is sequential) and every data step single-threaded and on every host core
    (threads over disjoint tokens or experts).  GB/s of the same algorithmic bytes."""
    smp = OracleSample(w, maxvio, seed, s_sample)
    cores = host_cores()
    b = smp.bytes()
    t0 = time.perf_counter()
    reps, el = _time_until(lambda: smp.o.plan(smp.cfg, smp.idx), min_s / 2)
    plan_us = el / reps * 1e6
    single, multi = {}, {}
    for name, fn in smp.kernels().items():
        r1, e1 = _time_until(lambda: fn(1), min_s)
        single[name] = b[name] * r1 / e1 / 1e9
        rn, en = _time_until(lambda: fn(cores), min_s)
        multi[name] = b[name] * rn / en / 1e9
    dc = b["dispatch"] + b["combine"]
    value = dc / (b["dispatch"] / multi["dispatch"] + b["combine"] / multi["combine"])
    value_1 = dc / (b["dispatch"] / single["dispatch"] + b["combine"] / single["combine"])
    return {"value": value, "unit": "GB/s", "cores": cores, "kind": "oracle",
            "single_thread_value": value_1, "plan_us_single_thread": plan_us,
            "single_thread": single, "all_cores": multi,
            "seconds": time.perf_counter() - t0,
            "sample": f"first {s_sample} of {w.S} tokens on each of the {w.R} ranks of the same "
                      f"seeded routing (maxvio {maxvio}), planned as one layer of S={s_sample}; "
                      f"expert gradient / weight rows cut to {smp.P} elements; every step of "
                      f"the layer timed single-threaded and on {cores} threads (disjoint tokens "
                      f"or experts), each repeated for >= {min_s:.1f} s; value = dispatch + "
                      f"combine on all {cores} threads"}


def run_reference(args, rank, world):
    """The reference arm: the CPU oracle on every host core, same metric and config, on a
    bounded sample of the workload per step."""
    if rank != 0:
        return 0
    w = WORKLOADS[args.workload]
    mv = args.maxvio if args.maxvio is not None else w.maxvio[0]
    s_sample = max(1, min(w.S, 64 if w.H >= 4096 else 256))
    import oracle
    R, E, K, H = w.R, w.E, w.K, w.H
    cores = host_cores()
    idx, alpha, realized = make_routing(R, E, K, w.S, mv, args.seed)
    gates = make_gates(R, w.S, K, args.seed)
    b = algorithmic_bytes(R, s_sample, K, H)
    cfg = oracle.Config(R=R, E=E, K=K, S=s_sample, H=H, budget=w.budget, mode=w.mode)
    times, plan_t = [], []
    deadline = time.perf_counter() + args.reference_budget_s
    done = 0
    for step in range(args.warmup + args.steps):
        # step s uses the s-th slice of s_sample tokens of every rank (wrapping)
        lo = (step * s_sample) % max(1, w.S - s_sample + 1)
        si = np.ascontiguousarray(idx[:, lo:lo + s_sample, :])
        sg = np.ascontiguousarray(gates[:, lo:lo + s_sample, :]).reshape(R * s_sample, K)
        x = make_x(R, s_sample, H, args.seed + step).reshape(R * s_sample, H)
        a = time.perf_counter()
        st, t = oracle.plan(cfg, si)
        m = time.perf_counter()
        slot_of = t["slot_of"]
        recv = np.zeros((R * int(t["nvs"][0]), H), np.uint16)
        parts = [p for p in np.array_split(np.arange(R * s_sample, dtype=np.int64), cores) if p.size]

        def disp(tk):
            t0, t1 = int(tk[0]), int(tk[-1]) + 1
            sub = oracle.Config(R=1, E=E, K=K, S=t1 - t0, H=H, budget=w.budget, mode=w.mode)
            oracle.dispatch(sub, slot_of[t0 * K:t1 * K], x[t0:t1], recv)

        _run_threads(disp, parts)
        _run_threads(lambda tk: oracle.combine(cfg, slot_of, recv, sg, tk), parts)
        e = time.perf_counter()
        if step >= args.warmup:
            times.append(e - m)
            plan_t.append(m - a)
            done += 1
        if time.perf_counter() > deadline and done >= 1:
            break
    gbs = (b["dispatch"] + b["combine"]) * done / sum(times) / 1e9
    sample = (f"per step {s_sample} tokens on each of the {R} ranks (a slice of the seeded "
              f"{args.workload} routing, maxvio {mv}), planned as one layer (single-threaded); "
              f"dispatch + combine in the C oracle on {cores} threads over disjoint tokens")
    line = {
        "impl": "reference", "metric": METRIC, "value": gbs, "unit": "GB/s", "n_gpus": world,
        "steps": done, "warmup": args.warmup, "ms_per_step": 1e3 * (sum(times) + sum(plan_t)) / done,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic", "config": workload_config(w, realized, alpha, world),
        "plan_us_per_layer": 1e6 * sum(plan_t) / done,
        "cpu_baseline": {"value": gbs, "unit": "GB/s", "cores": cores, "kind": "oracle",
                         "sample": sample, "sample_tokens_per_rank": s_sample},
        "e2e": {"value": gbs, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ main ---
def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(WORKLOADS))
    ap.add_argument("--maxvio", type=float, default=None)
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--impl", default="moonep", choices=["moonep", "reference"])
    ap.add_argument("--sweep", action="store_true", help="maxvio sweep of the workload shape")
    ap.add_argument("--compare-copy", action="store_true",
                    help="zero-copy dispatch+combine against the copy-through-buffer path")
    ap.add_argument("--scale-s", type=int, default=1, help="divide S (tokens/rank) by this (profiling)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-extra", action="store_true",
                    help="headline line only: no compact sweep, no decode workload")
    ap.add_argument("--extra-steps", type=int, default=20,
                    help="timed steps per point of the compact sweep and the decode runs")
    ap.add_argument("--reference-budget-s", type=float, default=120.0)
    args = ap.parse_args()

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        return run_reference(args, rank, world)

    import torch
    if not torch.cuda.is_available():
        print(json.dumps({"metric": METRIC, "error": "no CUDA device"}))
        return 1
    torch.cuda.set_device(local_rank)
    device = torch.device("cuda", local_rank)
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=device)
        pg = dist

    def barrier():
        if pg:
            pg.barrier()

    w = WORKLOADS[args.workload]
    if args.scale_s > 1:  # a smaller case of the same shape (profiling captures)
        import dataclasses
        w = dataclasses.replace(w, S=max(1, w.S // args.scale_s),
                                P=max(8, (w.P or 2048 * w.H) // args.scale_s))
    if args.sweep:
        return run_sweep(args, w, device)
    if args.compare_copy:
        return run_compare_copy(args, w, device)
    mv = args.maxvio if args.maxvio is not None else w.maxvio[0]
    layer = Layer(w, mv, args.seed + rank, device)
    total_ms, per, clocks, st = time_steps(layer, args.steps, args.warmup, barrier)
    b = layer.bytes()

    dc_ms = sum(per["dispatch"]) + sum(per["combine"])
    total_ms, dc_ms = max_over_ranks(pg, [total_ms, dc_ms], device)
    value = whole_job_gbs((b["dispatch"] + b["combine"]) * args.steps, world, dc_ms)
    peak, peak_src = hbm_peak()

    kern = {}
    per_total = sum(sum(ts) for ts in per.values())
    for name, ts in per.items():
        avg = sum(ts) / len(ts)
        kern[name] = {"ms": avg, "bytes": b[name], "GBs": b[name] / (avg * 1e-3) / 1e9,
                      "frac": b[name] / (avg * 1e-3) / 1e9 / peak, "share": sum(ts) / per_total}
    host_us = host_cost(layer, n=200 if w.name == DEFAULT_WORKLOAD else 500)
    b2b = time_back_to_back(layer)
    names = sorted(b2b)
    for name, ms in zip(names, max_over_ranks(pg, [b2b[n] for n in names], device)):
        kern[name].update({"b2b_ms": ms, "b2b_GBs": b[name] / (ms * 1e-3) / 1e9,
                           "b2b_frac": b[name] / (ms * 1e-3) / 1e9 / peak})
    kern["plan"].pop("frac")
    # the plan is a latency: its per-layer figure is the median over the steps
    kern["plan"]["ms_mean"] = kern["plan"]["ms"]
    kern["plan"]["ms"] = statistics.median(per["plan"])
    dom = max((k for k in kern if k != "plan"), key=lambda k: kern[k]["ms"])
    traffic = ncu_traffic(w.name if args.scale_s <= 1 else None, mv, args.seed).get(dom)
    roof = {"kernel": dom, "bound": "hbm", "achieved": kern[dom]["GBs"], "peak": peak,
            "unit": "GB/s", "frac": kern[dom]["GBs"] / peak, "traffic": traffic,
            "peak_source": f"{peak_src} copy bandwidth"}
    launches = len(layer.ops()) * args.steps
    headline_cfg = workload_config(w, layer.maxvio, layer.alpha, world, scaled=args.scale_s > 1)
    replicas = {"pieces": layer.n_piece, "local": layer.n_local, "remote": layer.n_remote,
                "experts_replicated": layer.n_rep_exp}

    rg_f32 = None
    if layer.train and not args.no_extra:
        rg_f32 = time_reduce_grad_f32(layer)
        rg_f32["ms"], rg_f32["b2b_ms"] = max_over_ranks(pg, [rg_f32["ms"], rg_f32["b2b_ms"]], device)
        for k in ("", "b2b_"):
            rg_f32[k + "GBs"] = rg_f32["bytes"] / (rg_f32[k + "ms"] * 1e-3) / 1e9
            rg_f32[k + "frac"] = rg_f32[k + "GBs"] / peak

    e2e = None
    if not args.no_e2e:
        n = min(args.steps, 20)
        ms, h2d, d2h = time_e2e(layer, n)
        ms = max_over_ranks(pg, [ms], device)[0]
        e2e = {"value": whole_job_gbs((b["dispatch"] + b["combine"]) * n, world, ms),
               "unit": "GB/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "ms_per_step": ms / n, "steps": n,
               "how": "inputs copied in and results read back every step, overlapped with "
                      "the previous/next step's compute (two buffer sets)"}

    sweep = decode = None
    if not args.no_extra and args.scale_s <= 1 and world == 1 and w.name == DEFAULT_WORKLOAD:
        ex_warm = max(3, min(args.warmup, 5))
        sweep = compact_sweep(layer, (0, 1), args.extra_steps, ex_warm)
        del layer
        torch.cuda.empty_cache()
        decode = decode_runs(device, args.extra_steps, ex_warm)
        torch.cuda.empty_cache()

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        cpu = oracle_baseline(w, mv, args.seed, s_sample=min(w.S, 128 if w.H >= 4096 else 256))

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": total_ms / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": headline_cfg,
            "pct_of_peak": {"measured": value / peak, "nominal_8TBs": value / NOMINAL_HBM_GBS},
            "plan_us_per_layer": kern["plan"]["ms"] * 1e3,
            "layer_us": 1e3 * (kern["plan"]["ms"] + kern["dispatch"]["ms"] + kern["combine"]["ms"]),
            "kernels": kern,
            "reduce_grad_f32": rg_f32,
            "replicas": replicas,
            "device_status": st,
            "roofline": roof,
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": launches,
            "host_us_per_call": host_us,
            "clocks": clocks,
            "sweep": sweep,
            "decode": decode,
        }
        print(json.dumps(line), flush=True)
    if pg:
        pg.barrier()
        pg.destroy_process_group()
    return 0


def run_compare_copy(args, w, device):
    """Forward layer with zero copy (moonep_dispatch / moonep_combine) against the
    zero_copy=False path (rows land in a comm buffer in arrival order, then a permute;
    permute back before combine).  Same results, same useful bytes."""
    import torch
    me = __import__("token_dispatch_moonep_b200")
    mv = args.maxvio if args.maxvio is not None else w.maxvio[0]
    layer = Layer(w, mv, args.seed, device, with_backward=False, host_inputs=False)
    c, T, K, N = layer.cfg, w.R * w.S, w.K, w.R * w.S * w.K
    comm = torch.empty_like(layer.recv)
    cidx = torch.empty(N + w.R, dtype=torch.int32, device=device)
    st = layer.status
    zc = [("dispatch", lambda: me.moonep_dispatch(c, layer.arena, layer.x, layer.recv, st)),
          ("combine", lambda: me.moonep_combine(c, layer.arena, layer.recv, layer.gates, layer.out,
                                                st))]
    vb = [("dispatch_via_buffer", lambda: me.moonep_dispatch_via_buffer(
              c, layer.arena, layer.x, comm, cidx, layer.recv, st)),
          ("combine_via_buffer", lambda: me.moonep_combine_via_buffer(
              c, layer.arena, layer.recv, layer.gates, cidx, comm, layer.out, st))]
    me.moonep_plan(c, layer.idx, layer.arena, layer.ws, st)
    res = {}
    for name, ops in (("zero_copy", zc), ("via_buffer", vb)):
        for _ in range(args.warmup):
            for _, fn in ops:
                fn()
        torch.cuda.synchronize()
        n = max(20, args.steps // 4)
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(ops) + 1)] for _ in range(n)]
        for i in range(n):
            ev[i][0].record()
            for j, (_, fn) in enumerate(ops):
                fn()
                ev[i][j + 1].record()
        torch.cuda.synchronize()
        per = {op: statistics.median(ev[i][j].elapsed_time(ev[i][j + 1]) for i in range(n))
               for j, (op, _) in enumerate(ops)}
        res[name] = per
    b = algorithmic_bytes(w.R, w.S, K, w.H)
    useful = b["dispatch"] + b["combine"]
    zc_ms, vb_ms = sum(res["zero_copy"].values()), sum(res["via_buffer"].values())
    print(json.dumps({"compare": "zero_copy vs via_buffer", "workload": w.name,
                      "maxvio": round(layer.maxvio, 4), "zero_copy_ms": res["zero_copy"],
                      "via_buffer_ms": res["via_buffer"],
                      "zero_copy_GBs": useful / (zc_ms * 1e-3) / 1e9,
                      "via_buffer_GBs": useful / (vb_ms * 1e-3) / 1e9,
                      "time_ratio": vb_ms / zc_ms, "device_status": int(st.item())}), flush=True)
    return 0


def run_sweep(args, w, device):
    """Plan µs and dispatch/combine GB/s per maxvio (5 seeds each), plus flatness.
    Forward only (plan + dispatch + combine), the per-layer time the pages plot."""
    layer = Layer(w, SWEEP_MAXVIO[0], 0, device, with_backward=False, host_inputs=False)
    targets = SWEEP_MAXVIO if args.maxvio is None else (args.maxvio,)
    res = compact_sweep(layer, (0, 1, 2, 3, 4), max(20, args.steps // 10), args.warmup, targets)
    for row in res["rows"]:
        print(json.dumps({k: v for k, v in row.items() if k != "seeds"}), flush=True)
    print(json.dumps(res), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
