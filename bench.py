#!/usr/bin/env python
"""Benchmark of the routed, block-quantized MoE FFN layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload decode|prefill|wide|cache]

One JSON line on rank 0.  Workloads (seeded synthetic inputs, see synthetic/):

* decode (default): the 30B-A3B-shaped layer (D=2048, E=128, top-8,
  F=768, Q4_0 experts, bf16 activations).  One step runs the layer at
  T = 1, 4 and 16 tokens (21 tokens), each call on another replica of the
  expert pool so that weights come from HBM, not L2 (6 replicas, 2 GB).
* prefill: the same shapes in Q8_0 at T = 8192 with a Zipf(1.1) router
  bias (skewed expert loads); 2 replicas of the pool.
* wide: E=512, top-10, F=512 Q4_0 plus a Q8_0 shared expert, routing
  logits from a temporal-locality trace, at T = 1 and T = 2048.
* cache: one token per step through a 40-layer stack of the decode layer in
  Q8_0 whose experts live in pinned host memory, 51 HBM slots (40%) per
  layer, misses copied on a side stream while the resident experts' FFN
  runs; reports tokens/s with routing read back from the GPU per layer
  (dependent) and with the ids known ahead (two_phase, lookahead), the hit
  rate, the copy bytes and the exposed copy time, against the same stack
  fully resident.

The default run (decode) prints the decode line with every other
configuration under "configs" (tiny, prefill, wide_t1, wide_t2048,
prefill_stream, cache), each with its own roofline, end-to-end number and
oracle baseline.  prefill_stream: the prefill layer stacked 8 deep with its
experts in pinned host memory, whole layers double-buffered into HBM.

Timing: W untimed steps, then K steps bracketed by a barrier and a device
synchronize, timed with CUDA events on the launching stream; max over
ranks.  Per-kernel times come from the library's own trace events recorded
inside the timed steps (moe_trace).  SM clocks and throttle reasons are
sampled through NVML while the timed steps run.  With N > 1 (torchrun)
every rank runs an independent replica of the layer (the layer does not
shard on one GPU's worth of work): weak scaling, no collective on the path.

``--impl reference`` times the CPU oracle (oracle/) on the host cores on a
bounded sample of the same workload: the only other place this file runs
the oracle besides the cpu_baseline leg.
"""
from __future__ import annotations

import argparse
import dataclasses
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synthetic as S  # noqa: E402

HBM_SPEC_GBS = 8000.0
TC_SPEC_TFLOPS = 2250.0


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """NVML sampling of SM clock and throttle reasons while a region runs."""

    REASONS = {
        "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4,
        "hw_slowdown": 0x8, "sync_boost": 0x10, "sw_thermal_slowdown": 0x20,
        "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80,
        "display_clock_setting": 0x100,
    }

    def __init__(self, device_index: int, period_s: float = 0.005):
        self.samples = []
        self.reasons = set()
        self.period = period_s
        self._stop = threading.Event()
        self.ok = False
        self.max_mhz = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # pragma: no cover - no NVML
            self.err = str(e)

    def _poll(self):
        nv = self.nv
        while True:
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for name, bit in self.REASONS.items():
                    if r & bit and name != "gpu_idle":
                        self.reasons.add(name)
            except Exception:
                pass
            if self._stop.wait(self.period):
                break

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._poll, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ------------------------------------------------------------ distributed
def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    import torch
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(v: float, world: int) -> float:
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# -------------------------------------------------------------- workloads
def _dev_x(L, torch):
    if L.cfg.x_dtype == "bf16":
        return torch.from_numpy(L.x_raw.view(np.int16)).cuda().view(torch.bfloat16)
    return torch.from_numpy(L.x_raw).cuda()


# tokens per call and pool replicas (enough that the pool copies together
# exceed L2, so every call reads its experts from HBM)
WORKLOADS = {
    "decode": ((1, 4, 16), 6),
    "tiny": ((4,), 1),
    "prefill": ((8192,), 2),
    "wide": ((1, 2048), 2),
    "wide_t1": ((1,), 2),
    "wide_t2048": ((2048,), 2),
}


# the other block types (the rest of the Standard family, the K-quants), each
# on the decode and prefill layer shapes: workload "<decode|prefill>_<type>",
# the configuration with its experts encoded in that type
STD_TYPES = ("q4_1", "q5_0", "q5_1", "q4_k", "q6_k")
STD_WORKLOADS = [f"{c}_{q}" for q in STD_TYPES for c in ("decode", "prefill")]
# 8-bit activations into every expert matmul (the W4A8 / W8A8 mode) on the
# decode layer: Q4_0 experts (W4A8) and the same weights in Q8_0 (W8A8)
A8_WORKLOADS = {"decode_a8": "q4_0", "decode_w8a8": "q8_0"}


def act_bits_of(name):
    return 8 if name in A8_WORKLOADS else 16


def workload_spec(name):
    """(layer configuration, T per call, pool replicas) of a workload name."""
    if name in WORKLOADS:
        Ts, replicas = WORKLOADS[name]
        return S.CONFIGS[name.split("_")[0]], Ts, replicas
    if name in A8_WORKLOADS:
        Ts, replicas = WORKLOADS["decode"]
        return dataclasses.replace(S.CONFIGS["decode"], qtype=A8_WORKLOADS[name], name=name), Ts, replicas
    base, qt = name.split("_", 1)
    if base not in ("decode", "prefill") or qt not in STD_TYPES:
        raise ValueError(f"unknown workload {name}")
    Ts, replicas = WORKLOADS[base]
    return dataclasses.replace(S.CONFIGS[base], qtype=qt, name=name), Ts, replicas


class Workload:
    """A list of layer calls making one step; replicas rotate per call."""

    def __init__(self, name: str, torch, moe, n_replicas=0, base=None):
        self.name = name
        self.torch, self.moe = torch, moe
        cfg, Ts, replicas = workload_spec(name)
        self.cfg = cfg
        if n_replicas:     # fewer replicas: a small case for profilers (weights may hit L2)
            replicas = int(n_replicas)
        self.Ts = Ts
        if base is None:
            base = S.make_layer(cfg, T=max(Ts))
        self.base = base
        self.inputs = {}
        for T in Ts:
            if T == base.x.shape[0]:
                self.inputs[T] = base
            else:
                self.inputs[T] = S.make_layer(cfg, T=T, experts=False)
                self.inputs[T].gate, self.inputs[T].up, self.inputs[T].down = base.gate, base.up, base.down
                self.inputs[T].shared = base.shared
        dev = lambda a: None if a is None else torch.from_numpy(np.ascontiguousarray(a)).cuda()
        g, u, d = dev(base.gate), dev(base.up), dev(base.down)
        self.expert_bytes = sum(S.expert_bytes(cfg.D, cfg.F, cfg.qtype))
        self.pool_bytes = g.numel() + u.numel() + d.numel()
        pools = [moe.ExpertPool(g, u, d, cfg.qtype)]
        for _ in range(replicas - 1):
            pools.append(moe.ExpertPool(g.clone(), u.clone(), d.clone(), cfg.qtype))
        shared = None
        if base.shared is not None:
            sg, su, sd = (dev(a) for a in base.shared)
            shared = moe.ExpertPool(sg, su, sd, cfg.shared_qtype)
            self.shared_bytes = sum(S.expert_bytes(cfg.D, cfg.shared_F, cfg.shared_qtype))
        else:
            self.shared_bytes = 0
        xdt = torch.bfloat16 if cfg.x_dtype == "bf16" else torch.float32
        ydt = torch.bfloat16 if cfg.y_dtype == "bf16" else torch.float32
        self.act_bits = act_bits_of(name)
        self.layers = [moe.Layer(p, cfg.D, cfg.F, cfg.E, cfg.k, max(Ts), w_router=dev(base.w_router),
                                 bias=dev(base.bias), shared=shared, shared_F=cfg.shared_F,
                                 renorm=cfg.renorm, x_dtype=xdt, y_dtype=ydt,
                                 act_bits=self.act_bits) for p in pools]
        self.x = {T: _dev_x(self.inputs[T], torch) for T in Ts}
        self.logits = {T: dev(self.inputs[T].logits) for T in Ts}
        self.y = {T: torch.empty((T, cfg.D), dtype=ydt, device="cuda") for T in Ts}
        self.xdt, self.ydt = xdt, ydt
        self.r = 0
        self.tokens_per_step = sum(Ts)
        self.calls_per_step = len(Ts)
        self.kernels_per_call = self._count_kernels()

    def _count_kernels(self):
        """Kernels one layer call launches (from a traced eager call)."""
        tr = self.moe.KernelTrace(n_calls=1)
        T = self.Ts[0]
        self.layers[0].forward(self.x[T], logits=self.logits[T], out=self.y[T], trace=tr)
        self.torch.cuda.synchronize()
        kinds = [k for k, _, _ in tr.calls[0]]
        # the decode FFN segment covers three kernels (gate/up, down, combine)
        return len(kinds) + 2 * kinds.count("ffn_decode")

    def step(self, trace=None, x=None, y=None, logits=None):
        for T in self.Ts:
            lay = self.layers[self.r]
            self.r = (self.r + 1) % len(self.layers)
            lay.forward(self.x[T] if x is None else x[T],
                        logits=self.logits[T] if logits is None else logits[T],
                        out=self.y[T] if y is None else y[T], trace=trace)

    def distinct_experts(self):
        out = {}
        for T in self.Ts:
            lay = self.layers[0]
            lay.forward(self.x[T], logits=self.logits[T], out=self.y[T])
            self.torch.cuda.synchronize()
            out[T] = int(np.unique(lay.ids[:T].cpu().numpy()).size)
        return out

    def algorithmic(self):
        """Algorithmic work of each call: HBM bytes of each traced segment
        (weights of the distinct experts once, activations in and out once)
        and tensor FLOPs."""
        cfg = self.cfg
        distinct = self.distinct_experts()
        gb, ub, db = S.expert_bytes(cfg.D, cfg.F, cfg.qtype)
        sg, su, sd = (S.expert_bytes(cfg.D, cfg.shared_F, cfg.shared_qtype) if cfg.shared_F
                      else (0, 0, 0))
        act = 2 if cfg.x_dtype == "bf16" else 4
        yb = 2 if cfg.y_dtype == "bf16" else 4
        per_call = {}
        for T in self.Ts:
            n = distinct[T]
            rows = T * cfg.k + (T if cfg.shared_F else 0)
            fl_gu = 2.0 * T * cfg.k * 2 * cfg.D * cfg.F + (2.0 * T * 2 * cfg.D * cfg.shared_F)
            fl_dn = 2.0 * T * cfg.k * cfg.D * cfg.F + (2.0 * T * cfg.D * cfg.shared_F)
            x_b = T * cfg.D * act
            h_b = rows * cfg.F * 2                       # fp16 hidden rows
            seg = {
                "ffn_decode": n * (gb + ub + db) + self.shared_bytes + x_b + T * cfg.D * yb,
                "gateup": n * (gb + ub) + sg + su + x_b + h_b,
                "down": n * db + sd + h_b + T * cfg.D * yb,
                "route": (cfg.D * cfg.E * 4 if self.inputs[T].w_router is not None else T * cfg.E * 4) + x_b,
            }
            per_call[T] = {"distinct": n, "seg_bytes": seg, "flops": fl_gu + fl_dn,
                           "seg_flops": {"gateup": fl_gu, "down": fl_dn, "ffn_decode": fl_gu + fl_dn},
                           "weight_bytes": n * (gb + ub + db) + self.shared_bytes}
        return per_call


# ------------------------------------------------------------- our arm
def capture_graph(torch, fn, n):
    """Capture n calls of fn (library launches only) into one CUDA graph."""
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for _ in range(n):
            fn()
    return g


class _Eager:
    def __init__(self, fn, n):
        self.fn, self.n = fn, n

    def replay(self):
        for _ in range(self.n):
            self.fn()


def gpu_lead(torch):
    """A short device-side spin (about 0.5 ms, torch's bounded sleep kernel)
    queued just before a timed region's start event: the host then submits
    the graph while the GPU is still busy, so the region starts with the
    graph's first kernel instead of with host launch latency."""
    torch.cuda._sleep(1_000_000)


class E2EPipe:
    """End-to-end steps with the host copies overlapped: step i's input copy
    (pinned host -> device) runs on its own stream while step i-1 computes,
    and step i's result copy (device -> pinned host) on a third stream while
    step i+1 computes, through two device buffers each way.  Every copy of
    every step lies inside the region timed around run(), which ends when
    the last result has reached host memory (the side streams join the
    calling stream there)."""

    def __init__(self, torch, wl, xh, lh):
        self.torch, self.wl, self.xh, self.lh = torch, wl, xh, lh
        self.s_in, self.s_out = torch.cuda.Stream(), torch.cuda.Stream()
        self.xd = [{T: torch.empty_like(wl.x[T]) for T in wl.Ts} for _ in range(2)]
        self.ld = [{T: None if lh[T] is None else torch.empty_like(wl.logits[T]) for T in wl.Ts}
                   for _ in range(2)]
        self.yd = [{T: torch.empty_like(wl.y[T]) for T in wl.Ts} for _ in range(2)]
        self.yh = {T: torch.empty(wl.y[T].shape, dtype=wl.ydt).pin_memory() for T in wl.Ts}
        self.with_logits = wl.logits[wl.Ts[0]] is not None

    def run(self, n):
        torch, wl = self.torch, self.wl
        main = torch.cuda.current_stream()
        fork = torch.cuda.Event()
        fork.record(main)
        self.s_in.wait_event(fork)
        self.s_out.wait_event(fork)
        x_in, done, y_out = [None, None], [None, None], [None, None]
        for i in range(n):
            b = i % 2
            with torch.cuda.stream(self.s_in):
                if done[b] is not None:          # step i-2 has read its inputs
                    self.s_in.wait_event(done[b])
                for T in wl.Ts:
                    self.xd[b][T].copy_(self.xh[T], non_blocking=True)
                    if self.lh[T] is not None:
                        self.ld[b][T].copy_(self.lh[T], non_blocking=True)
                x_in[b] = torch.cuda.Event()
                x_in[b].record(self.s_in)
            main.wait_event(x_in[b])
            if y_out[b] is not None:             # step i-2's result is out
                main.wait_event(y_out[b])
            wl.step(x=self.xd[b], y=self.yd[b], logits=self.ld[b] if self.with_logits else None)
            done[b] = torch.cuda.Event()
            done[b].record(main)
            with torch.cuda.stream(self.s_out):
                self.s_out.wait_event(done[b])
                for T in wl.Ts:
                    self.yh[T].copy_(self.yd[b][T], non_blocking=True)
                y_out[b] = torch.cuda.Event()
                y_out[b].record(self.s_out)
        main.wait_event(x_in[(n - 1) % 2])
        main.wait_event(y_out[(n - 1) % 2])


def measure_layer(wl, steps, warmup, world, local, peaks, no_graph=False, cpu=True,
                  cpu_seconds=10.0):
    """Timed pass, traced pass, end-to-end pass of one workload; returns the
    JSON fields of its line (or sub-object)."""
    torch, moe = wl.torch, wl.moe
    algo = wl.algorithmic()
    stream = torch.cuda.current_stream()
    # eager calls first (first-use set-up), then the steps as CUDA graphs:
    # the decode layer is a handful of short kernels and would otherwise wait
    # on the host's launch path (--no-graph launches every step eagerly)
    wl.step()
    torch.cuda.synchronize()
    trace = moe.KernelTrace(n_calls=steps * wl.calls_per_step)
    if no_graph:
        g_warm, g_plain = _Eager(wl.step, warmup), _Eager(wl.step, steps)
        g_traced = _Eager(lambda: wl.step(trace=trace), steps)
    else:
        g_warm = capture_graph(torch, wl.step, warmup)
        g_plain = capture_graph(torch, wl.step, steps)
        g_traced = capture_graph(torch, lambda: wl.step(trace=trace), steps)
    g_warm.replay()
    torch.cuda.synchronize()

    # ---- timed region: K steps (one graph replay), events at its ends only:
    # an event recorded between two kernels ends the programmatic launch
    # overlap of the next kernel with the previous one, so the per-kernel
    # trace runs as a second pass of the same K steps (below)
    barrier(world)
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local, period_s=0.0005) as clk:
        gpu_lead(torch)
        t0.record(stream)
        g_plain.replay()
        t1.record(stream)
        torch.cuda.synchronize()
    barrier(world)
    ms_step = max_over_ranks(t0.elapsed_time(t1) / steps, world)

    # ---- traced pass: the same K steps with the library's trace events
    # between its kernels (per-kernel durations for the roofline)
    barrier(world)
    torch.cuda.synchronize()
    u0, u1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    gpu_lead(torch)
    u0.record(stream)
    g_traced.replay()
    u1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    ms_traced = max_over_ranks(u0.elapsed_time(u1) / steps, world)
    durs = trace.durations()

    # ---- end to end: pinned host x (and logits) -> device, layer, device
    # -> pinned host y, all inside the timed region
    xh = {T: wl.x[T].cpu().pin_memory() for T in wl.Ts}
    yh = {T: torch.empty(wl.y[T].shape, dtype=wl.ydt).pin_memory() for T in wl.Ts}
    xd = {T: torch.empty_like(wl.x[T]) for T in wl.Ts}
    h2d = sum(xh[T].numel() * xh[T].element_size() for T in wl.Ts)
    d2h = sum(yh[T].numel() * yh[T].element_size() for T in wl.Ts)
    lh = {T: None if wl.logits[T] is None else wl.logits[T].cpu().pin_memory() for T in wl.Ts}
    ld = {T: None if wl.logits[T] is None else torch.empty_like(wl.logits[T]) for T in wl.Ts}
    h2d += sum(lh[T].numel() * 4 for T in wl.Ts if lh[T] is not None)

    def e2e_step():
        for T in wl.Ts:
            xd[T].copy_(xh[T], non_blocking=True)
            if lh[T] is not None:
                ld[T].copy_(lh[T], non_blocking=True)
        wl.step(x=xd, logits=ld if wl.logits[wl.Ts[0]] is not None else None)
        for T in wl.Ts:
            yh[T].copy_(wl.y[T], non_blocking=True)

    pipe = E2EPipe(torch, wl, xh, lh)

    class _Run:
        def __init__(self, fn):
            self.fn = fn

        def replay(self):
            self.fn()

    def graph_of(fn):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            fn()
        return g

    if no_graph:
        for _ in range(warmup):
            e2e_step()
        g_e2e = _Eager(e2e_step, steps)
        pipe.run(warmup)
        g_pipe = _Run(lambda: pipe.run(steps))
    else:
        g_e2e = capture_graph(torch, e2e_step, steps)
        capture_graph(torch, e2e_step, warmup).replay()
        graph_of(lambda: pipe.run(warmup)).replay()
        g_pipe = graph_of(lambda: pipe.run(steps))
    torch.cuda.synchronize()

    def timed(g):
        barrier(world)
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        gpu_lead(torch)
        a.record(stream)
        g.replay()
        b.record(stream)
        torch.cuda.synchronize()
        ms = max_over_ranks(a.elapsed_time(b) / steps, world)
        barrier(world)
        return ms

    serial_ms = timed(g_e2e)
    e2e_ms = timed(g_pipe)
    # the pipelined steps compute what the plain ones do (same inputs, same
    # deterministic kernels, replicas of the same weights): the last result
    # that reached host memory equals the device output of the plain steps
    for T in wl.Ts:
        if not torch.equal(pipe.yh[T], wl.y[T].cpu()):
            raise RuntimeError(f"{wl.name}: pipelined end-to-end result differs at T={T}")

    tokens = wl.tokens_per_step * world
    out = {
        "value": round(tokens / (ms_step / 1e3), 2),
        "unit": "tokens/s",
        "ms_per_step": round(ms_step, 5),
        "config": config_of(wl),
        "roofline": roofline(wl, algo, durs, peaks, steps),
        "kernels_ms": {k: round(sum(v) / len(v), 5) for k, v in sorted(durs.items())},
        "kernels_pass": {"ms_per_step": round(ms_traced, 5),
                         "note": "kernels_ms and the roofline come from a second pass of the same "
                                 "K steps with trace events between the library's kernels; those "
                                 "events cut the launch overlap, so that pass runs slower than the "
                                 "timed one"},
        "gpu_launches": wl.kernels_per_call * wl.calls_per_step * steps,
        "e2e": {"value": round(tokens / (e2e_ms / 1e3), 2), "unit": "tokens/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "serial": round(tokens / (serial_ms / 1e3), 2),
                "how": "pinned host inputs copied in and results copied out every step, on "
                       "their own streams, overlapping the neighbouring steps' layer calls; "
                       "serial: each step's copies and calls one after another on one stream"},
        "clocks": clk.summary(),
        "launch": "eager" if no_graph else "cuda-graph replay",
    }
    if cpu:
        out["cpu_baseline"] = cpu_baseline(wl, cpu_seconds)
    return out


def dtype_of(cfg, act_bits=16):
    if act_bits == 8:
        return f"{cfg.qtype} weights, 8-bit activation blocks, int32 accumulate"
    return f"{cfg.qtype} weights, bf16 activations, fp32 accumulate"


def config_of(wl):
    cfg = wl.cfg
    c = {"workload": f"{wl.name}: MoE layer D={cfg.D} E={cfg.E} top-{cfg.k} F={cfg.F} "
                     f"{cfg.qtype.upper()}"
                     + (f" + shared F={cfg.shared_F} {cfg.shared_qtype.upper()}" if cfg.shared_F else "")
                     + f", T per call {list(wl.Ts)}",
         "tokens_per_step": wl.tokens_per_step,
         "l2": f"{len(wl.layers)} rotating replicas of the expert pool "
               f"({wl.pool_bytes / 1e6:.0f} MB each): weights come from HBM"}
    return c


# the dominant kernel's bound per workload: the tensor-core GEMM at T=8192
# (about 960 FLOP per weight byte, above the B200's ridge of about 250), HBM
# for everything else (the wide layer at T=2048 does about 140 FLOP per byte)
TENSOR_BOUND = {"prefill"}


def roofline(wl, algo, durs, peaks, steps):
    """Roofline of the dominant traced segment over the timed steps."""
    tot = {k: sum(v) for k, v in durs.items()}
    dom = max(tot, key=tot.get)
    launches = len(durs[dom])
    avg_ms = tot[dom] / launches
    flops_step = sum(algo[T]["seg_flops"].get(dom, 0.0) for T in wl.Ts)
    bytes_step = sum(algo[T]["seg_bytes"].get(dom, 0) for T in wl.Ts)
    tflops = flops_step * steps / (tot[dom] / 1e3) / 1e12
    gbs = bytes_step * steps / (tot[dom] / 1e3) / 1e9
    if wl.name.split("_")[0] in TENSOR_BOUND and dom in ("gateup", "down"):
        bound, achieved, peak, unit, spec = "tensor", tflops, peaks["bf16_tflops"], "TFLOP/s", TC_SPEC_TFLOPS
        psrc = "bf16_tflops burst (fp16 operands run at the bf16 rate)"
        work = flops_step
    else:
        bound, achieved, peak, unit, spec = "hbm", gbs, peaks["hbm_gbs"], "GB/s", HBM_SPEC_GBS
        psrc = "hbm_gbs"
        work = bytes_step
    r = {"kernel": dom, "bound": bound, "achieved": round(achieved, 2), "peak": peak,
         "unit": unit, "frac": round(achieved / peak, 4), "frac_of_spec": round(achieved / spec, 4),
         "algorithmic_per_launch": round(work / wl.calls_per_step, 1),
         "avg_launch_ms": round(avg_ms, 5),
         "per_T": {str(T): {"work": algo[T]["seg_flops" if bound == "tensor" else "seg_bytes"].get(dom),
                            "distinct_experts": algo[T]["distinct"],
                            # launches run in T order within a step
                            "avg_ms": round(sum(durs[dom][i::len(wl.Ts)]) /
                                            max(1, len(durs[dom][i::len(wl.Ts)])), 5)}
                   for i, T in enumerate(wl.Ts)},
         "peak_source": f"{peaks['source']} {psrc}",
         "traffic": ncu_traffic(dom, wl.name)}
    if flops_step and bound == "hbm":
        r["tensor_frac_of_measured"] = round(tflops / peaks["bf16_tflops"], 4)
    if bound == "tensor":
        r["frac_of_sustained"] = round(tflops / peaks["bf16_tflops_sustained"], 4)
        r["hbm_gbs_at_algorithmic_bytes"] = round(gbs, 1)
    # the other FFN kernels of the step, for context
    others = {}
    for k in ("gateup", "down", "ffn_decode"):
        if k in tot and k != dom:
            fl = sum(algo[T]["seg_flops"].get(k, 0.0) for T in wl.Ts) * steps / (tot[k] / 1e3) / 1e12
            by = sum(algo[T]["seg_bytes"].get(k, 0) for T in wl.Ts) * steps / (tot[k] / 1e3) / 1e9
            others[k] = {"avg_launch_ms": round(tot[k] / len(durs[k]), 5), "tflops": round(fl, 2),
                         "gbs": round(by, 1)}
    if others:
        r["other_kernels"] = others
    return r


# the source files whose code runs in each traced segment's kernels
SEGMENT_SOURCES = {"ffn_decode": ("ffn_decode.cu", "sm100.cuh", "moe_internal.cuh"),
                   "gateup": ("ffn_prefill.cu", "sm100.cuh", "moe_internal.cuh"),
                   "down": ("ffn_prefill.cu", "sm100.cuh", "moe_internal.cuh")}


def segment_sha(kernel):
    import hashlib
    h = hashlib.sha256()
    src = os.path.join(ROOT, "quantized_routed_expert_top_b200", "csrc")
    for f in SEGMENT_SOURCES.get(kernel, ()):
        h.update(open(os.path.join(src, f), "rb").read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel, workload):
    """dram read+write bytes per launch from the committed ncu summary, only
    while the segment's kernel sources still hash to what was profiled."""
    p = os.path.join(ROOT, "profiles", "traffic.md")
    if not os.path.exists(p) or kernel not in SEGMENT_SOURCES:
        return None
    sha = segment_sha(kernel)
    for line in open(p):
        if line.startswith("traffic:"):
            kv = dict(x.split("=", 1) for x in line.split()[1:])
            if kv.get("kernel") == kernel and kv.get("workload") == workload and kv.get("src_sha") == sha:
                return float(kv["bytes_per_launch"])
    return None


# ------------------------------------------------------------- cache arm
def h2d_probe(torch, nbytes=1 << 30):
    """Pinned host -> device copy bandwidth in GB/s: one 1 GiB copy after a warm-up."""
    h = torch.empty(nbytes, dtype=torch.uint8, pin_memory=True)
    d = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    s = torch.cuda.Stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(s):
        d.copy_(h, non_blocking=True)
        e0.record(s)
        d.copy_(h, non_blocking=True)
        e1.record(s)
    s.synchronize()
    gbs = nbytes / (e0.elapsed_time(e1) / 1e3) / 1e9
    del h, d
    return gbs


CACHE_MODES = {
    "dependent": "each layer routes on the GPU, its ids come back to the host (a 32-byte "
                 "copy and a wait), the host LRU requests them, then the layer runs in two "
                 "calls: the resident experts' FFN while the misses copy, then the copied "
                 "experts' FFN and the combine",
    "two_phase": "the host knows each layer's ids from the trace ahead of the GPU (no wait "
                 "per layer); each layer runs in two calls around the copy wait as above",
    "lookahead": "ids from the trace ahead of the GPU; each layer waits for all its copies, "
                 "then runs in one call",
}


class CacheStack:
    """A stack of the Q8_0 decode layer whose experts live in pinned host
    memory; each layer keeps a fraction of its experts in HBM slots (LRU) and
    copies misses on a side stream.  One step = one token through the stack,
    routed by per-layer temporal-locality traces; the residual stream is
    x <- bf16(x + y) after each layer."""

    def __init__(self, torch, moe, n_layers, n_tokens):
        cfg = S.CONFIGS["cache"]
        self.torch, self.moe, self.cfg = torch, moe, cfg
        E, k, D, F = cfg.E, cfg.k, cfg.D, cfg.F
        self.n_layers, self.n_tokens = n_layers, n_tokens
        self.n_slots = int(math.floor(S.CACHE_FRACTION * E))
        # one layer's experts, the same bytes for every layer (the copy and
        # kernel costs do not depend on the values; drawing 40 pools would
        # take minutes of host time)
        self.pool_np = S.gen_expert_pool(cfg.seed, E, D, F, cfg.qtype, cfg.expert_std)
        pin = lambda a: torch.empty(a.shape, dtype=torch.uint8, pin_memory=True).copy_(torch.from_numpy(a))
        self.host = [[pin(a) for _ in range(n_layers)] for a in self.pool_np]
        self.sets, lg = [], []
        for l in range(n_layers):
            logits, sets = S.locality_trace(np.random.default_rng([cfg.seed, l]), n_tokens, E, k)
            lg.append(logits)
            self.sets.append(sets)
        self.logits_host = np.ascontiguousarray(np.stack(lg, axis=1))   # [tokens, layers, E]
        self.logits = torch.from_numpy(self.logits_host).cuda()
        _, raw = S.gen_activations(np.random.default_rng([cfg.seed, 0x70]), 1, D, "bf16")
        self.x0 = torch.from_numpy(raw.view(np.int16)).cuda().view(torch.bfloat16)
        self.x = self.x0.clone()
        self.y = torch.empty_like(self.x)
        self.copy_stream = torch.cuda.Stream()
        self.cache = moe.ExpertCache(*self.host, cfg.qtype, self.n_slots, self.copy_stream)
        self.layers = [moe.Layer(self.cache.pools[l], D, F, E, k, 1) for l in range(n_layers)]
        self.ids_host = torch.empty((n_layers, k), dtype=torch.int32, pin_memory=True)
        self.ids_ready = torch.cuda.Event()
        self.resident = None

    def use_cache(self, cache):
        """Route the stack through another cache over the same host pools."""
        cfg = self.cfg
        self.cache = cache
        self.layers = [self.moe.Layer(cache.pools[l], cfg.D, cfg.F, cfg.E, cfg.k, 1)
                       for l in range(self.n_layers)]

    def make_resident(self):
        """The same stack with every expert resident in HBM (one pool per layer)."""
        torch, moe, cfg = self.torch, self.moe, self.cfg
        pools = []
        for l in range(self.n_layers):
            g, u, d = (torch.from_numpy(a).cuda() for a in self.pool_np)
            pools.append(moe.ExpertPool(g, u, d, cfg.qtype))
        self.resident = [moe.Layer(p, cfg.D, cfg.F, cfg.E, cfg.k, 1) for p in pools]

    def token(self, t, mode="dependent", logits=None):
        moe = self.moe
        stream = self.torch.cuda.current_stream()
        lg = self.logits[t] if logits is None else logits
        for l in range(self.n_layers):
            if mode == "resident":
                self.resident[l].forward(self.x, logits=lg[l:l + 1], out=self.y)
                self.x.add_(self.y)
                continue
            lay, c = self.layers[l], self.cache
            if mode == "dependent":
                # route on the GPU; the ids come back before the request
                lay.forward(self.x, logits=lg[l:l + 1], out=self.y, phases=moe.PHASE_ROUTE)
                self.ids_host[l].copy_(lay.ids[0], non_blocking=True)
                self.ids_ready.record(stream)
                self.ids_ready.synchronize()
                c.request(l, self.ids_host[l].numpy(), stream=stream)
                lay.forward(self.x, logits=lg[l:l + 1], out=self.y, mask=c.hit_mask(l),
                            phases=moe.PHASE_FFN | moe.PHASE_SHARED)
            elif mode == "two_phase":
                c.request(l, self.sets[l][t], stream=stream)
                lay.forward(self.x, logits=lg[l:l + 1], out=self.y, mask=c.hit_mask(l),
                            phases=moe.PHASE_ROUTE | moe.PHASE_FFN | moe.PHASE_SHARED)
            else:   # lookahead, one call after the copies
                c.request(l, self.sets[l][t], stream=stream)
                c.sync(l, stream=stream)
                lay.forward(self.x, logits=lg[l:l + 1], out=self.y)
                c.release(l, stream=stream)
                self.x.add_(self.y)
                continue
            c.sync(l, stream=stream)
            lay.forward(self.x, logits=lg[l:l + 1], out=self.y, mask=c.miss_mask(l),
                        phases=moe.PHASE_FFN | moe.PHASE_COMBINE)
            c.release(l, stream=stream)
            self.x.add_(self.y)

    def kernels_per_layer_call(self):
        tr = self.moe.KernelTrace(n_calls=1)
        self.resident[0].forward(self.x0, logits=self.logits[0, 0:1], out=self.y, trace=tr)
        self.torch.cuda.synchronize()
        kinds = [k for k, _, _ in tr.calls[0]]
        return len(kinds) + 2 * kinds.count("ffn_decode")


def oracle_cache_sample(pool_np, logits_host, n_layers, n_sample):
    """The oracle on one token through the first n_sample layers of the stack."""
    import oracle
    oracle.build()
    cfg = S.CONFIGS["cache"]
    g, u, d = pool_np
    x0, _ = S.gen_activations(np.random.default_rng([cfg.seed, 0x70]), 1, cfg.D, "bf16")
    x = x0.astype(np.float32)
    t = time.perf_counter()
    for l in range(n_sample):
        ids, gw = oracle.select(logits_host[0, l][None, :].astype(np.float64), cfg.k, cfg.renorm)
        y = oracle.layer(x, ids, gw, g, u, d, cfg.qtype, cfg.F)
        x = S.bf16_bits_to_f32(S.f32_to_bf16_bits((x + np.asarray(y, np.float32)).astype(np.float32)))
    dt = time.perf_counter() - t
    return n_sample / (dt * n_layers), dt


def cache_layers(args):
    cfg = S.CONFIGS["cache"]
    gb, ub, db = S.expert_bytes(cfg.D, cfg.F, cfg.qtype)
    layer_bytes = cfg.E * (gb + ub + db)
    want = args.cache_layers or S.CACHE_LAYERS
    ram = os.sysconf("SC_PAGE_SIZE") * os.sysconf("SC_PHYS_PAGES")
    fit = int(0.5 * ram // layer_bytes)
    if fit >= want:
        return want, None
    return max(1, fit), (f"{want} layers need {want * layer_bytes / 1e9:.1f} GB of pinned host "
                         f"memory; this host has {ram / 1e9:.0f} GB, so {max(1, fit)} layers")


# tokens run before each point of the cache-size sweep: the first point
# starts from an empty pool (about 60 misses per token fill 2970 slots in
# about 50 tokens, most of them within 30), later ones settle after a resize
SWEEP_FILL = (30, 8)


def measure_cache(args, steps, warmup, world, local, peaks, cpu=True):
    import torch
    import quantized_routed_expert_top_b200 as moe
    n_layers, reduced = cache_layers(args)
    modes = ("dependent", "two_phase", "lookahead")
    n_tok = (warmup + steps * (len(modes) + 1) + 5 * max(4, min(steps, 12)) + SWEEP_FILL[0] +
             4 * SWEEP_FILL[1] + 1)
    st = CacheStack(torch, moe, n_layers, n_tok)
    st.make_resident()
    kpl = st.kernels_per_layer_call()
    pcie = h2d_probe(torch)
    stream = torch.cuda.current_stream()
    ev = lambda: torch.cuda.Event(enable_timing=True)
    cursor = [0]

    def timed(mode, n):
        st.x.copy_(st.x0)
        torch.cuda.synchronize()
        h0, m0, b0 = st.cache.stats()
        x0 = st.cache.exposed_ns()
        barrier(world)
        e0, e1 = ev(), ev()
        with ClockSampler(local, period_s=0.002) as clk:
            e0.record(stream)
            for _ in range(n):
                st.token(cursor[0], mode)
                cursor[0] += 1
            e1.record(stream)
            torch.cuda.synchronize()
        h1, m1, b1 = st.cache.stats()
        x1 = st.cache.exposed_ns()
        return e0.elapsed_time(e1), (h1 - h0, m1 - m0, b1 - b0, x1 - x0), clk

    timed("dependent", warmup)               # warm the cache and the kernels
    res = {}
    for mode in modes:
        ms, (hits, misses, nbytes, exp_ns), clk = timed(mode, steps)
        res[mode] = {"tokens_per_s": round(steps * world / (max_over_ranks(ms, world) / 1e3), 3),
                     "ms_per_token": round(ms / steps, 4),
                     "hit_rate": round(hits / max(1, hits + misses), 4),
                     "misses_per_token": round(misses / steps, 3),
                     "bytes_copied_per_token": int(nbytes // steps),
                     "copy_gbs": round(nbytes / (ms / 1e3) / 1e9, 2),
                     "exposed_copy_ms_per_token": round(exp_ns / 1e6 / steps, 4),
                     "how": CACHE_MODES[mode]}
        if mode == "dependent":
            clk_dep, ms_dep, bytes_dep = clk, ms, nbytes
    # the pages' cache-size experiment: one global LRU over every layer's
    # experts, resized at run time (no restart, host pools untouched) from
    # 58% to 10% of all experts; tokens/s and hit rate with dependent routing
    sweep = {}
    fracs = (0.58, 0.40, 0.30, 0.20, 0.10)
    total = n_layers * st.cfg.E
    per_layer_cache = st.cache
    gcache = moe.ExpertCache(*st.host, st.cfg.qtype, int(round(fracs[0] * total)), st.copy_stream,
                             global_slots=int(round(fracs[0] * total)))
    st.use_cache(gcache)
    n_sweep = max(4, min(steps, 12))
    for i, f in enumerate(fracs):
        cap = int(round(f * total))
        gcache.resize(cap, stream=stream)
        fill = SWEEP_FILL[0] if i == 0 else SWEEP_FILL[1]
        if cursor[0] + n_sweep + fill > n_tok:
            cursor[0] = 0
        timed("dependent", fill)          # fill (the first point starts empty) or settle
        ms, (hits, misses, nbytes, exp_ns), _ = timed("dependent", n_sweep)
        sweep[f"{int(round(f * 100))}%"] = {
            "slots": cap, "tokens_per_s": round(n_sweep / (ms / 1e3), 3),
            "hit_rate": round(hits / max(1, hits + misses), 4),
            "misses_per_token": round(misses / n_sweep, 3),
            "exposed_copy_ms_per_token": round(exp_ns / 1e6 / n_sweep, 4)}
    base = sweep["58%"]["tokens_per_s"]
    for v in sweep.values():
        v["rel_to_58%"] = round(v["tokens_per_s"] / base, 4)
    gcache.close()
    st.use_cache(per_layer_cache)
    saved = cursor[0]
    cursor[0] = 0
    ms_res = 0.0
    st.x.copy_(st.x0)
    torch.cuda.synchronize()
    e0, e1 = ev(), ev()
    e0.record(stream)
    for t in range(steps):
        st.token(t, "resident")
    e1.record(stream)
    torch.cuda.synchronize()
    ms_res = e0.elapsed_time(e1)
    cursor[0] = saved

    # end to end (dependent mode): each token's x and its per-layer trace
    # logits come from pinned host memory, its output goes back to pinned host
    xh = st.x0.cpu().pin_memory()
    yh = torch.empty_like(xh).pin_memory()
    lh = torch.from_numpy(st.logits_host).pin_memory()
    lbuf = torch.empty_like(st.logits[0])
    n_e2e = min(steps, n_tok - cursor[0])
    torch.cuda.synchronize()
    e0, e1 = ev(), ev()
    e0.record(stream)
    for _ in range(n_e2e):
        t = cursor[0]
        cursor[0] += 1
        st.x.copy_(xh, non_blocking=True)
        lbuf.copy_(lh[t], non_blocking=True)
        st.token(t, "dependent", logits=lbuf)
        yh.copy_(st.x, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize()
    ms_e2e = max_over_ranks(e0.elapsed_time(e1), world)

    dep = res["dependent"]
    achieved = bytes_dep / (ms_dep / 1e3) / 1e9
    cfg = st.cfg
    out = {
        "value": dep["tokens_per_s"], "unit": "tokens/s",
        "ms_per_step": dep["ms_per_token"],
        "config": {"workload": f"cache: one token per step through a {n_layers}-layer stack of the "
                               f"MoE layer D={cfg.D} E={cfg.E} top-{cfg.k} F={cfg.F} Q8_0, experts "
                               f"in pinned host memory, {st.n_slots} HBM slots per layer (LRU), "
                               f"dependent routing (value); two_phase / lookahead modes beside it",
                   "layers": n_layers, "slots_per_layer": st.n_slots,
                   "l2": "each step streams its misses from host memory; the resident comparison "
                         "keeps one pool per layer in HBM",
                   **({"reduced": reduced} if reduced else {})},
        "roofline": {"kernel": "expert miss copies (host to device)", "bound": "pcie",
                     "achieved": round(achieved, 2), "peak": round(pcie, 2), "unit": "GB/s",
                     "frac": round(achieved / pcie, 4),
                     "peak_source": "pinned 1 GiB host-to-device copy measured in this run",
                     "traffic": None},
        "modes": res,
        "global_lru_resize_sweep": {
            "how": "one LRU over all layers' experts (global mode), capacity changed at run time "
                   "with moe_cache_resize between points; dependent routing; pages: 58% -> 40% "
                   "costs about 10%, below 20% a sharp drop (RTX 5090, whole-model decode)",
            "points": sweep},
        "resident_tokens_per_s": round(steps / (ms_res / 1e3), 3),
        "gpu_launches": kpl * n_layers * steps,
        "e2e": {"value": round(n_e2e * world / (ms_e2e / 1e3), 3), "unit": "tokens/s",
                "h2d_bytes_per_step": xh.numel() * xh.element_size() + lh[0].numel() * 4,
                "d2h_bytes_per_step": yh.numel() * yh.element_size()},
        "clocks": clk_dep.summary(),
        "launch": "eager (the host LRU runs at every layer call)",
    }
    if cpu:
        ns = min(n_layers, 4)
        v, dt = oracle_cache_sample(st.pool_np, st.logits_host, n_layers, ns)
        out["cpu_baseline"] = {"value": round(v, 5), "unit": "tokens/s", "cores": os.cpu_count() or 1,
                               "kind": "oracle",
                               "sample": f"one token through {ns} of the {n_layers} layers (fp64), "
                                         f"{dt:.1f} s, scaled to the whole stack"}
    st.cache.close()
    return out


# --------------------------------------------------- streamed prefill arm
STREAM_LAYERS = 8


def measure_prefill_stream(torch, moe, base, steps, warmup, peaks, cpu=True):
    """The prefill layer (T=8192, Q8_0) stacked STREAM_LAYERS deep with every
    layer's experts in pinned host memory, streamed a whole layer at a time
    into two device buffers while the previous layer computes."""
    cfg = base.cfg
    gb, ub, db = S.expert_bytes(cfg.D, cfg.F, cfg.qtype)
    layer_bytes = cfg.E * (gb + ub + db)
    ram = os.sysconf("SC_PAGE_SIZE") * os.sysconf("SC_PHYS_PAGES")
    n_layers = max(2, min(STREAM_LAYERS, int(0.3 * ram // layer_bytes)))
    pin = lambda a: torch.empty(a.shape, dtype=torch.uint8, pin_memory=True).copy_(torch.from_numpy(a))
    # one drawn pool's bytes for every layer (the copy and kernel costs do not
    # depend on the values)
    host = [[pin(a) for _ in range(n_layers)] for a in (base.gate, base.up, base.down)]
    st = moe.LayerStreamer(*host, cfg.qtype, torch.cuda.Stream())
    dev = lambda a: None if a is None else torch.from_numpy(np.ascontiguousarray(a)).cuda()
    T = base.x.shape[0]
    lay = moe.Layer(moe.ExpertPool(dev(base.gate), dev(base.up), dev(base.down), cfg.qtype),
                    cfg.D, cfg.F, cfg.E, cfg.k, T, w_router=dev(base.w_router), bias=dev(base.bias))
    resident_pool = lay.pool
    x0 = _dev_x(base, torch)
    x = x0.clone()
    y = torch.empty_like(x)
    stream = torch.cuda.current_stream()

    def stack_pass(streamed):
        if streamed:
            st.prefetch(0)
            st.prefetch(1)
        for l in range(n_layers):
            lay.pool = st.acquire(l, stream=stream) if streamed else resident_pool
            lay.forward(x, out=y)
            if streamed:
                st.release(l, stream=stream)
                if l + 2 < n_layers:
                    st.prefetch(l + 2)
            x.add_(y)

    def timed(streamed, n):
        x.copy_(x0)
        torch.cuda.synchronize()
        b0, e0n = st.stats()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(n):
            stack_pass(streamed)
        e1.record(stream)
        torch.cuda.synchronize()
        b1, e1n = st.stats()
        return e0.elapsed_time(e1), b1 - b0, e1n - e0n

    passes = max(1, min(steps, 3))
    tr = moe.KernelTrace(n_calls=1)
    lay.forward(x0, out=y, trace=tr)
    torch.cuda.synchronize()
    kpl = len(tr.calls[0])                # kernels per layer call
    timed(True, 1)
    with ClockSampler(0, period_s=0.002) as clk:
        ms, nbytes, exp_ns = timed(True, passes)
    timed(False, 1)
    ms_res, _, _ = timed(False, passes)
    pcie = h2d_probe(torch)
    # end to end: the prompt's activations from pinned host memory, the last
    # layer's output back to pinned host memory, inside the timed region
    xh = x0.cpu().pin_memory()
    yh = torch.empty_like(xh).pin_memory()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(passes):
        x.copy_(xh, non_blocking=True)
        stack_pass(True)
        yh.copy_(x, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize()
    ms_e2e = e0.elapsed_time(e1)
    tok = T * n_layers * passes
    out = {
        "value": round(tok / (ms / 1e3), 1), "unit": "tokens/s",
        "ms_per_step": round(ms / passes / n_layers, 4),
        "config": {"workload": f"prefill_stream: the prefill layer (T={T}, D={cfg.D}, E={cfg.E}, "
                               f"top-{cfg.k}, F={cfg.F}, {cfg.qtype.upper()}) stacked {n_layers} deep, "
                               f"every layer's {layer_bytes / 1e6:.0f} MB of experts in pinned host "
                               f"memory, copied a whole layer at a time into two device buffers "
                               f"while the previous layer computes; tokens/s per layer",
                   "layers": n_layers, "passes": passes},
        "roofline": {"kernel": "layer copies (host to device)", "bound": "pcie",
                     "achieved": round(nbytes / (ms / 1e3) / 1e9, 2), "peak": round(pcie, 2),
                     "unit": "GB/s", "frac": round(nbytes / (ms / 1e3) / 1e9 / pcie, 4),
                     "peak_source": "pinned 1 GiB host-to-device copy measured in this run",
                     "traffic": None},
        "exposed_copy_ms_per_layer": round(exp_ns / 1e6 / passes / n_layers, 4),
        "resident_ms_per_layer": round(ms_res / passes / n_layers, 4),
        "resident_tokens_per_s": round(tok / (ms_res / 1e3), 1),
        "gpu_launches": kpl * n_layers * passes,
        "e2e": {"value": round(tok / (ms_e2e / 1e3), 1), "unit": "tokens/s",
                "h2d_bytes_per_step": xh.numel() * xh.element_size(),
                "d2h_bytes_per_step": yh.numel() * yh.element_size()},
        "clocks": clk.summary(),
    }
    if cpu:
        import oracle
        oracle.build()
        t0 = time.perf_counter()
        m = 16
        _, ids, g = oracle.route(base.x[:m], base.w_router, base.bias, cfg.k, cfg.renorm)
        oracle.layer(base.x[:m], ids, g, base.gate, base.up, base.down, cfg.qtype, cfg.F)
        dt = time.perf_counter() - t0
        out["cpu_baseline"] = {"value": round(m / dt, 4), "unit": "tokens/s",
                               "cores": os.cpu_count() or 1, "kind": "oracle",
                               "sample": f"{m} tokens through one layer (route + layer, fp64; the "
                                         f"oracle reads host memory, no streaming), {dt:.1f} s"}
    st.close()
    del host
    return out


def _line(out, args, world, cfg, peaks):
    line = {"metric": "MoE-layer tokens/s", "value": out["value"], "unit": out["unit"],
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": out["ms_per_step"], "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": dtype_of(cfg, act_bits_of(args.workload)),
            "data": "synthetic (seeded; random-init experts in ggml Standard blocks, no checkpoint)"}
    for k, v in out.items():
        if k not in line:
            line[k] = v
    line["peaks"] = peaks
    return line


# the other configurations of the default run: (key, workload)
EXTRA = [("tiny", "tiny"), ("prefill", "prefill"), ("wide_t1", "wide_t1"),
         ("wide_t2048", "wide_t2048")]


def std_base(cfg_name, qtype, pool):
    """Inputs of the decode or prefill configuration (T = its largest call)
    over a given expert pool."""
    cfg, Ts, _ = workload_spec(f"{cfg_name}_{qtype}")
    L = S.make_layer(cfg, T=max(Ts), experts=False)
    L.gate, L.up, L.down = pool
    return L


def std_base_a8(name):
    """Inputs of the decode configuration over its expert pool encoded in
    the 8-bit-activation workload's type."""
    cfg, Ts, _ = workload_spec(name)
    L = S.make_layer(cfg, T=max(Ts))
    return L


def measure_std_types(torch, moe, steps, warmup, world, local, peaks, no_graph, cpu):
    """The decode and prefill layers with experts in Q4_1, Q5_0, Q5_1, Q4_K
    and Q6_K: one expert pool per type (the decode shape's weights, encoded
    in that type), each workload with its own roofline and end-to-end
    number (Q6_K prefill converts its pool to fp16 rows for the tensor-core
    GEMM)."""
    out = {}
    for qt in STD_TYPES:
        cfg = S.CONFIGS["decode"]
        pool = S.gen_expert_pool(cfg.seed, cfg.E, cfg.D, cfg.F, qt, cfg.expert_std)
        for c in ("decode", "prefill"):
            name = f"{c}_{qt}"
            w = Workload(name, torch, moe, base=std_base(c, qt, pool))
            out[name] = measure_layer(w, steps, warmup, world, local, peaks, no_graph, cpu=cpu,
                                      cpu_seconds=3.0)
            del w
            torch.cuda.empty_cache()
        del pool
    return out


def run_ours(args, world, rank, local):
    import torch
    import quantized_routed_expert_top_b200 as moe
    from quantized_routed_expert_top_b200 import build as B
    if rank == 0 or not os.path.exists(moe.LIB_PATH):
        B.build()
    barrier(world)
    moe.lib()
    peaks = measured_peaks()
    with_cpu = rank == 0 and world == 1 and not args.no_cpu_baseline
    if args.workload == "cache":
        out = measure_cache(args, args.steps, args.warmup, world, local, peaks, cpu=with_cpu)
        if rank == 0:
            print(json.dumps(_line(out, args, world, S.CONFIGS["cache"], peaks)), flush=True)
        return
    wl = Workload(args.workload, torch, moe, args.replicas)
    out = measure_layer(wl, args.steps, args.warmup, world, local, peaks, args.no_graph, cpu=with_cpu)
    line = _line(out, args, world, wl.cfg, peaks)
    del wl
    if args.workload == "decode" and not args.no_extra and world == 1:
        # every other configuration, each with its own roofline, end-to-end
        # number and oracle baseline (fewer steps: the decode line is the
        # headline, these keep the whole run within a few minutes)
        steps = max(5, min(args.steps, 20))
        line["configs"] = {}
        bases = {}
        for key, name in EXTRA:
            cfg_name = name.split("_")[0]
            if cfg_name not in bases:      # one expert pool per configuration
                T_big = max(max(WORKLOADS[n][0]) for _, n in EXTRA if n.split("_")[0] == cfg_name)
                bases[cfg_name] = S.make_layer(S.CONFIGS[cfg_name], T=T_big)
            w = Workload(name, torch, moe, base=bases[cfg_name])
            line["configs"][key] = measure_layer(w, steps, args.warmup, world, local, peaks,
                                                 args.no_graph, cpu=with_cpu, cpu_seconds=6.0)
            del w
            torch.cuda.empty_cache()
        for name in sorted(A8_WORKLOADS):
            w = Workload(name, torch, moe, base=std_base_a8(name))
            line["configs"][name] = measure_layer(w, steps, args.warmup, world, local, peaks,
                                                  args.no_graph, cpu=with_cpu, cpu_seconds=3.0)
            line["configs"][name]["dtype"] = dtype_of(w.cfg, 8)
            del w
            torch.cuda.empty_cache()
        line["configs"]["standard_types"] = measure_std_types(torch, moe, steps, args.warmup,
                                                              world, local, peaks, args.no_graph,
                                                              with_cpu)
        torch.cuda.empty_cache()
        line["configs"]["prefill_stream"] = measure_prefill_stream(
            torch, moe, bases["prefill"], args.steps, args.warmup, peaks, cpu=with_cpu)
        torch.cuda.empty_cache()
        line["configs"]["cache"] = measure_cache(args, max(5, min(args.steps, 16)), args.warmup,
                                                 world, local, peaks, cpu=with_cpu)
    if rank == 0:
        print(json.dumps(line), flush=True)


# ------------------------------------------------------------ CPU oracle
def oracle_step_fn(wl_inputs, cfg, Ts, frac=1.0, act_bits=16):
    import oracle
    oracle.build()
    run = oracle.layer_a8 if act_bits == 8 else oracle.layer

    def step():
        n = 0
        for T in Ts:
            L = wl_inputs[T]
            if L.logits is not None:
                ids, g = oracle.select(L.logits, cfg.k, cfg.renorm)
            else:
                _, ids, g = oracle.route(L.x, L.w_router, L.bias, cfg.k, cfg.renorm)
            m = max(1, int(round(T * frac)))
            toks = np.arange(m, dtype=np.int32)
            run(L.x, ids, g, L.gate, L.up, L.down, cfg.qtype, cfg.F, shared=L.shared,
                tokens=toks, shared_qtype=cfg.shared_qtype)
            n += m
        return n
    return step


def cpu_baseline(wl, seconds=10.0):
    """The oracle as it stands, on the host cores, on a bounded sample."""
    cores = os.cpu_count() or 1
    frac = 1.0 if max(wl.Ts) <= 16 else 32.0 / max(wl.Ts)
    step = oracle_step_fn(wl.inputs, wl.cfg, wl.Ts, frac, wl.act_bits)
    t = time.perf_counter()
    n = step()
    dt = time.perf_counter() - t
    reps = 1
    while time.perf_counter() - t < seconds and reps < 20:
        n += step()
        reps += 1
    dt = time.perf_counter() - t
    return {"value": round(n / dt, 4), "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"{reps} oracle step(s) of {wl.name} on {n // reps} tokens each "
                      f"(route + layer, fp64, OpenMP over tokens), {dt:.1f} s wall"}


def run_reference_cache(args, world):
    """Reference arm of the cache workload: the oracle on one token through a
    sample of the stack's layers per step, scaled to the whole stack (the
    oracle has no cache: it computes the same layers from the host pool)."""
    cfg = S.CONFIGS["cache"]
    n_layers, reduced = cache_layers(args)
    pool = S.gen_expert_pool(cfg.seed, cfg.E, cfg.D, cfg.F, cfg.qtype, cfg.expert_std)
    lg = np.ascontiguousarray(np.stack(
        [S.locality_trace(np.random.default_rng([cfg.seed, l]), 1, cfg.E, cfg.k)[0] for l in range(n_layers)],
        axis=1))
    ns = 1
    for _ in range(max(0, args.warmup - 1)):
        oracle_cache_sample(pool, lg, n_layers, ns)
    t = time.perf_counter()
    for _ in range(args.steps):
        oracle_cache_sample(pool, lg, n_layers, ns)
    dt = time.perf_counter() - t
    value = args.steps * ns / (dt * n_layers)
    cores = os.cpu_count() or 1
    out = {"metric": "MoE-layer tokens/s", "value": round(value, 5), "unit": "tokens/s",
           "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
           "ms_per_step": round(dt / args.steps * 1e3, 3), "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "f64 (oracle)",
           "data": "synthetic (seeded)", "impl": "reference",
           "config": {"workload": f"cache: same {n_layers}-layer stack as the default arm; each step "
                                  f"one token through {ns} layer, scaled to the stack",
                      **({"reduced": reduced} if reduced else {})},
           "cpu_baseline": {"value": round(value, 5), "unit": "tokens/s", "cores": cores,
                            "kind": "oracle",
                            "sample": f"one token through {ns} of {n_layers} layers per step, "
                                      f"{args.steps} steps"},
           "e2e": {"value": round(value, 5), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                   "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


def run_reference(args, world, rank):
    """Reference arm: the CPU oracle, timed on the host cores."""
    if rank != 0:
        return
    name = args.workload
    if name == "cache":
        run_reference_cache(args, world)
        return
    cfg, Ts, _ = workload_spec(name)
    base = S.make_layer(cfg, T=max(Ts))
    inputs = {max(Ts): base}
    for T in Ts:
        if T not in inputs:
            inputs[T] = S.make_layer(cfg, T=T, experts=False)
            inputs[T].gate, inputs[T].up, inputs[T].down = base.gate, base.up, base.down
            inputs[T].shared = base.shared
    # size the per-step sample so that warmup + steps end within ~3 minutes
    small = max(Ts) <= 16
    step = oracle_step_fn(inputs, cfg, Ts, 1.0 if small else 16.0 / max(Ts), act_bits_of(name))
    t = time.perf_counter()
    n1 = step()
    t1 = time.perf_counter() - t
    budget = 150.0 / max(1, args.steps + args.warmup)
    frac = 1.0
    if t1 > budget:
        frac = max(budget / t1, 1.0 / n1)
    total = sum(Ts)
    step = oracle_step_fn(inputs, cfg, Ts, frac * (1.0 if small else 16.0 / max(Ts)), act_bits_of(name))
    for _ in range(max(0, args.warmup - 1)):
        step()
    t = time.perf_counter()
    n = 0
    for _ in range(args.steps):
        n += step()
    dt = time.perf_counter() - t
    value = n / dt
    cores = os.cpu_count() or 1
    out = {"metric": "MoE-layer tokens/s", "value": round(value, 4), "unit": "tokens/s",
           "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
           "ms_per_step": round(dt / args.steps * 1e3, 3), "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "f64 (oracle)",
           "data": "synthetic (seeded)", "impl": "reference",
           "config": {"workload": f"{name}: same layer as the default arm; each step a "
                                  f"sample of {n // args.steps} of its {total} tokens"},
           "cpu_baseline": {"value": round(value, 4), "unit": "tokens/s", "cores": cores,
                            "kind": "oracle",
                            "sample": f"{n // args.steps} tokens per step, {args.steps} steps"},
           "e2e": {"value": round(value, 4), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                   "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS) + STD_WORKLOADS + sorted(A8_WORKLOADS) + ["cache"],
                    default="decode",
                    help="the workload of the line (decode also reports every other one under "
                         "'configs' unless --no-extra)")
    ap.add_argument("--cache-layers", type=int, default=0,
                    help="layers of the cache stack (default: 40, fewer if host memory is short)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true")
    ap.add_argument("--replicas", type=int, default=0,
                    help="pool replicas (default: the workload's; fewer only for profiling)")
    ap.add_argument("--no-graph", action="store_true",
                    help="launch the steps eagerly instead of replaying CUDA graphs")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        run_reference(args, world, rank)
        return
    world, rank, local = dist_setup()
    try:
        run_ours(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
