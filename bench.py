#!/usr/bin/env python
"""Benchmark of the routed int4 MoE layer on B200.

One step = one pass of the whole hot path over one batch: route (router GEMV + top-k) and
batch union, gate/up int4 GEMV + SwiGLU, down int4 GEMV + routing-weighted combine with
the shared expert.  Default workload: the GLM-5.2-shaped layer decoding one token
(hidden 6144, 256 experts of intermediate 2048, top-8 + 1 shared, fp32 activations).

Timing: W untimed warm-up steps, then exactly K timed steps.  L2 is flushed (a write of
twice its size) before every step, outside the timed intervals; each step is bracketed by
CUDA events on the launching stream, and the kernels inside it by further events.  The
value is tokens/s over all ranks (replicas: one independent layer per GPU), with the
max over ranks of the summed step time.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints one JSON line (rank 0).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MoE-layer tokens/s; expert-weight HBM GB/s as fraction of B200 peak (decode)"
DEFAULT_WORKLOAD = "glm52_moe_h6144_i2048_e256_k8_t1"
FALLBACK_HBM_GBS = 6650.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--pool", type=int, default=64, help="distinct token batches rotated over")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--steady", action="store_true",
                    help="also time back-to-back calls (no flush) rotating over weight copies "
                         "that together hold at least 3x L2")
    ap.add_argument("--formats-only", action="store_true",
                    help="print only the weight-container comparison (int4 gs64 / int8 gs64 / int4 per-row / "
                         "int2 gs64): speed at the GLM shape and error against fp32 weights at hidden 1024")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the other configurations' lines (run by default at N=1)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--api", default="layer", choices=["layer", "calls"],
                    help="timed step: one coli_moe_layer call per layer, or the separate "
                         "route_union / gate_up / down calls")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--ref-seconds", type=float, default=60.0,
                    help="--impl reference: time budget of the timed oracle steps")
    ap.add_argument("--n-experts", type=int, default=0,
                    help="profiling captures only: keep the first N routed experts")
    ap.add_argument("--tokens", type=int, default=0,
                    help="profiling captures only: tokens per step instead of the workload's")
    return ap.parse_args()


# ------------------------------------------------------------------------------------
# helpers
# ------------------------------------------------------------------------------------

def max_over_ranks(values, world, device="cpu"):
    """Each value's maximum over the ranks (one all-reduce; NCCL with device tensors, gloo
    with CPU tensors).  Timings of a multi-GPU run are the slowest rank's."""
    import torch
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if world > 1:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return [float(v) for v in t.cpu().tolist()]


def job_rate(units_per_rank, world, total_ms):
    """Whole-job throughput: the units every rank processed over the slowest rank's time."""
    return units_per_rank * world / (total_ms * 1e-3)


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def source_hash(files):
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


KERNEL_SOURCES = {
    "gate_up": ["int4_routed_expert_gemv_b200/csrc/gemv.cu",
                "int4_routed_expert_gemv_b200/csrc/gemv.cuh",
                "int4_routed_expert_gemv_b200/csrc/common.cuh"],
    "down": ["int4_routed_expert_gemv_b200/csrc/gemv.cu",
             "int4_routed_expert_gemv_b200/csrc/gemv.cuh",
             "int4_routed_expert_gemv_b200/csrc/common.cuh"],
    "route_union": ["int4_routed_expert_gemv_b200/csrc/route.cu",
                    "int4_routed_expert_gemv_b200/csrc/select.cuh",
                    "int4_routed_expert_gemv_b200/csrc/union.cuh"],
    "fused_moe_kernel": ["int4_routed_expert_gemv_b200/csrc/fused.cu",
                         "int4_routed_expert_gemv_b200/csrc/fused.cuh",
                         "int4_routed_expert_gemv_b200/csrc/common.cuh"],
}


def recorded_traffic(kernel, workload):
    """DRAM bytes per launch from an ncu capture, if the kernel is unchanged since."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(workload, {}).get(kernel)
    if not e or e.get("source_hash") != source_hash(KERNEL_SOURCES[kernel]):
        return None
    return float(e["dram_bytes_per_launch"])


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the GPU works."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.rows = []
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu_id, f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "20"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 9:
                self.rows.append((time.time(), parts))

    def stop(self):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self, t0, t1):
        rows = [r for (t, r) in self.rows if t0 - 0.05 <= t <= t1 + 0.05] or [r for _, r in self.rows]
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}

        def num(v):
            try:
                return float(v)
            except ValueError:
                return None
        sm = [num(r[1]) for r in rows if num(r[1]) is not None]
        mx = [num(r[2]) for r in rows if num(r[2]) is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows)}


# ------------------------------------------------------------------------------------
# our implementation
# ------------------------------------------------------------------------------------

def run_ours(args, rank, world, local_rank):
    import torch

    from int4_routed_expert_gemv_b200 import binding as B
    from int4_routed_expert_gemv_b200 import build as builder
    from int4_routed_expert_gemv_b200 import synth

    if rank == 0 or world == 1:
        builder.build()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    wl = synth.WORKLOADS[args.workload]
    if args.n_experts:
        import dataclasses
        shp = dataclasses.replace(wl.shape, n_experts=args.n_experts)
        wl = dataclasses.replace(wl, shape=shp, name=f"{wl.name}_first{args.n_experts}experts")
    if args.tokens:
        import dataclasses
        wl = dataclasses.replace(wl, tokens=args.tokens, name=f"{wl.name}_as_t{args.tokens}")
    if wl.x_dtype == "bf16":
        return run_prefill(args, wl, rank, world, dev)
    s = wl.shape
    T = wl.tokens
    H, I, E, k = s.hidden, s.inter, s.n_experts, s.top_k
    NL = wl.layers
    stack = NL > 1

    dims = B.make_dims(H, I, E, k, s.n_shared)
    layers = []
    for l in range(NL):
        ex = synth.experts_tensor(s, wl.seed, l, device=dev)
        sh = synth.shared_tensor(s, wl.seed, l, device=dev)
        wr = torch.from_numpy(synth.router_weight(s, wl.seed, l)).to(dev)
        bias = torch.from_numpy(synth.zipf_bias(E)).to(dev) if wl.zipf else None
        layers.append(dict(experts=ex, shared=sh, wr=wr, bias=bias,
                           weights=B.make_weights(wr, bias, ex, sh, s.stride)))
    bufs = B.LayerBuffers(dims, T, device=dev)
    gamma = torch.ones(H, dtype=torch.float32, device=dev)
    x_work = torch.empty(T, H, dtype=torch.float32, device=dev)
    n_work = torch.empty(T, H, dtype=torch.float32, device=dev)

    R = args.pool
    xs_host = [torch.from_numpy(synth.activations(s, wl.seed, T, 1000 + i)).pin_memory()
               for i in range(R)]
    xs = [x.to(dev) for x in xs_host]
    y_host = torch.empty(T, H, dtype=torch.float32).pin_memory()
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    flush_buf = torch.empty(2 * l2 // 4 + 1024, dtype=torch.float32, device=dev)
    flush_read = torch.zeros(2 * l2 // 4 + 1024, dtype=torch.float32, device=dev)
    flush_sink = torch.empty(1, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    slots = 4 if stack else 3          # kernels timed per layer
    # decode batches (T <= 4) through the layer API run the fused kernel: one launch per
    # layer, or one launch for the whole stack (coli_moe_stack)
    fused = args.api == "layer" and T <= 4
    y_stack = torch.empty(T, H, dtype=torch.float32, device=dev)
    stack_w = [L_["weights"] for L_ in layers]

    def layer_calls(l, x_in, ev, e0):
        """One layer; ev[e0 .. e0+slots] bracket its launches."""
        L_ = layers[l]
        if ev:
            ev[e0].record()
        if stack:
            B.check(B.coli_rmsnorm(H, T, x_in, gamma, 1e-5, n_work), "rmsnorm")
            if ev:
                ev[e0 + 1].record()
            act, res, y = n_work, x_in, x_in
        else:
            act, res, y = x_in, None, bufs.y
        e = e0 + (1 if stack else 0)
        B.check(B.coli_moe_route_union(dims, L_["wr"], L_["bias"], act, T, bufs.idx, bufs.w, None,
                                       bufs.union_ids, bufs.n_union, bufs.offsets, bufs.assign,
                                       bufs.ws), "route_union")
        if ev:
            ev[e + 1].record()
        B.check(B.coli_moe_gate_up(dims, L_["weights"], act, T, bufs.union_ids, bufs.n_union,
                                   bufs.offsets, bufs.assign, bufs.ws), "gate_up")
        if ev:
            ev[e + 2].record()
        B.check(B.coli_moe_down(dims, L_["weights"], T, bufs.w, bufs.union_ids, bufs.n_union,
                                bufs.offsets, bufs.assign, res, y, bufs.ws), "down")
        if ev:
            ev[e + 3].record()

    def step(i, ev=None):
        if stack:
            x_work.copy_(xs[i % R])
            for l in range(NL):
                layer_calls(l, x_work, ev, l * (slots + 1))
        else:
            layer_calls(0, xs[i % R], ev, 0)

    def layer_api(l, x_in):
        """One layer through the single-call API (routing fused into the expert launches)."""
        if stack:
            B.check(B.coli_rmsnorm(H, T, x_in, gamma, 1e-5, n_work), "rmsnorm")
            act, res, y = n_work, x_in, x_in
        else:
            act, res, y = x_in, None, bufs.y
        B.check(B.coli_moe_layer(dims, layers[l]["weights"], act, T, bufs.idx, bufs.w, None,
                                 bufs.union_ids, bufs.n_union, bufs.offsets, bufs.assign, res, y,
                                 bufs.ws), "coli_moe_layer")

    one_layer = layer_api if args.api == "layer" else (lambda l, x_in: layer_calls(l, x_in, None, 0))

    def step_coarse(i, ev):
        """The step with events only around it (no event nodes between kernels, so
        consecutive launches keep their programmatic dependency)."""
        ev[0].record()
        if stack and fused:
            B.check(B.coli_moe_stack(dims, stack_w, [gamma] * NL, 1e-5, xs[i % R], T, None, y_stack,
                                     bufs.ws), "coli_moe_stack")
        elif stack:
            x_work.copy_(xs[i % R])
            for l in range(NL):
                one_layer(l, x_work)
        else:
            one_layer(0, xs[i % R])
        ev[1].record()

    # union size of every (batch, layer), deterministic, for the byte counts
    n_union = []
    for i in range(R):
        row = []
        if stack:
            x_work.copy_(xs[i])
        for l in range(NL):
            layer_calls(l, x_work if stack else xs[i], None, 0)
            row.append(int(bufs.n_union[0].item()))
        n_union.append(row)

    def flush():
        # write 2x L2, then read another 2x L2: our data is evicted and L2 is left holding
        # clean lines, so no write-back of the flush lands inside the timed interval
        flush_buf.zero_()
        torch.sum(flush_read, dim=0, keepdim=True, out=flush_sink)

    # The timed steps run as CUDA graphs (flush + the step's launches, with event-record
    # nodes around each launch), so the GPU never waits for the host to enqueue work.
    nev = NL * (slots + 1)

    def capture(first, n, coarse=False):
        evs = [[torch.cuda.Event(enable_timing=True, external=True) for _ in range(2 if coarse else nev)]
               for _ in range(n)]
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for i in range(n):
                flush()
                if coarse:
                    step_coarse(first + i, evs[i])
                else:
                    step(first + i, evs[i])
        return g, evs

    gpu_id = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    sampler = ClockSampler(gpu_id)
    sampler.start()
    time.sleep(0.2)
    K = args.steps
    G = min(K, 128 if not stack else 8)
    chunks = [(c, min(G, K - c)) for c in range(0, K, G)]
    graphs = {}
    for (c, n) in chunks:
        if n not in graphs:
            graphs[n] = capture(args.warmup, n, coarse=True)
    if args.warmup:
        gw, _ = capture(0, args.warmup)
        gw.replay()
    torch.cuda.synchronize(dev)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    # timed: K steps, events around each whole step (the flush stays outside)
    step_rows = []
    t0 = time.time()
    for (c, n) in chunks:
        g, evs = graphs[n]
        g.replay()
        torch.cuda.synchronize(dev)
        for i in range(n):
            step_rows.append(evs[i][0].elapsed_time(evs[i][1]))
    t1 = time.time()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    del graphs
    # per-kernel breakdown (for the roofline): the same steps with an event around every
    # launch; these events serialise the launches, so their sum is a little above the step
    Kb = min(K, G)
    gb, evb = capture(args.warmup, Kb)
    gb.replay()
    torch.cuda.synchronize(dev)
    seg_rows = []
    for i in range(Kb):
        per = np.zeros(slots)
        for l in range(NL):
            e0 = l * (slots + 1)
            for j in range(slots):
                per[j] += evb[i][e0 + j].elapsed_time(evb[i][e0 + j + 1])
        seg_rows.append(per)
    del gb
    time.sleep(0.1)
    sampler.stop()
    clocks = sampler.summary(t0, t1)
    seg = np.array(seg_rows)
    if stack:
        seg = seg[:, 1:]                 # route_union, gate_up, down (rmsnorm reported apart)
        rms_ms = np.array(seg_rows)[:, 0]
    step_ms = np.array(step_rows)
    total_ms = float(step_ms.sum())
    st, bits = B.coli_moe_read_status(bufs.ws)
    if st != B.COLI_OK:
        raise SystemExit(f"device status {bits:#x} after the timed region")

    # e2e: host buffers through the public calls, copies inside the timed interval
    e2e = None
    if not args.no_e2e:
        ev2 = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
        xin = torch.empty_like(xs[0])

        def e2e_step(i):
            xin.copy_(xs_host[i % R], non_blocking=True)
            if stack and fused:
                B.check(B.coli_moe_stack(dims, stack_w, [gamma] * NL, 1e-5, xin, T, None, y_stack, bufs.ws))
                y_host.copy_(y_stack, non_blocking=True)
            elif stack:
                for l in range(NL):
                    B.check(B.coli_rmsnorm(H, T, xin, gamma, 1e-5, n_work))
                    B.check(B.coli_moe_layer(dims, layers[l]["weights"], n_work, T, bufs.idx,
                                             bufs.w, None, bufs.union_ids, bufs.n_union,
                                             bufs.offsets, bufs.assign, xin, xin, bufs.ws))
                y_host.copy_(xin, non_blocking=True)
            else:
                B.check(B.coli_moe_layer(dims, layers[0]["weights"], xin, T, bufs.idx, bufs.w,
                                         None, bufs.union_ids, bufs.n_union, bufs.offsets,
                                         bufs.assign, None, bufs.y, bufs.ws))
                y_host.copy_(bufs.y[:T], non_blocking=True)
        for i in range(min(args.warmup, 5)):
            flush()
            e2e_step(i)
        torch.cuda.synchronize(dev)
        for i in range(K):
            flush()
            ev2[i][0].record(stream)
            e2e_step(i)
            ev2[i][1].record(stream)
        torch.cuda.synchronize(dev)
        e2e_ms = float(sum(ev2[i][0].elapsed_time(ev2[i][1]) for i in range(K)))
        e2e = (e2e_ms, T * H * 4, T * H * 4)

    total_ms, e2e_ms = max_over_ranks([total_ms, e2e[0] if e2e else 0.0], world, dev)
    if rank != 0:
        return None

    # algorithmic bytes (per step, summed over the layers of the step)
    blob = s.blob_bytes
    gu_bytes_expert = 2 * (I * H // 2) + 2 * (I * H // 64) * 2
    dn_bytes_expert = H * I // 2 + H * (I // 64) * 2
    nu = np.array([sum(n_union[(args.warmup + i) % R]) for (c, n) in chunks for i in range(n)],
                  dtype=np.float64)
    units = nu + NL * s.n_shared
    x_bytes = T * H * 4
    h_bytes = (T * k + T * s.n_shared) * I * 4
    route_bytes = NL * (E * H * 4 + x_bytes + T * E * 4)
    gu_bytes = units * gu_bytes_expert + NL * (x_bytes + h_bytes)
    dn_bytes = units * dn_bytes_expert + NL * (h_bytes + T * H * 4)
    step_bytes = route_bytes + units * blob + NL * (x_bytes + 2 * h_bytes + T * H * 4)
    peak, peak_kind = measured_peaks()
    kern = {
        "route_union": (seg[:, 0], np.full(Kb, float(route_bytes))),
        "gate_up": (seg[:, 1], gu_bytes[:Kb]),
        "down": (seg[:, 2], dn_bytes[:Kb]),
    }
    kernels = {}
    for name, (ms, by) in kern.items():
        avg_ms = float(ms.mean())
        gbs = float(by.sum() / (ms.sum() * 1e-3) / 1e9)
        kernels[name] = {"avg_us": round(avg_ms * 1e3, 3), "bytes_per_launch": float(by.mean()),
                         "gb_s": round(gbs, 1), "frac": round(gbs / peak, 4),
                         "share": round(float(ms.sum() / seg.sum()), 4)}
    if stack:
        kernels["rmsnorm"] = {"avg_us": round(float(rms_ms.mean()) * 1e3, 3),
                              "share": round(float(rms_ms.sum() / step_ms.sum()), 4)}
    dom = max((n for n in kernels if n != "rmsnorm"), key=lambda n: kernels[n]["share"])
    if fused:
        # the timed step is one launch of the fused kernel: its bytes over its duration
        fgbs = float(step_bytes.sum() / (total_ms * 1e-3) / 1e9)
        kernels = {"fused_moe_kernel": {"avg_us": round(total_ms / K * 1e3, 3),
                                        "bytes_per_launch": float(step_bytes.mean()),
                                        "gb_s": round(fgbs, 1), "frac": round(fgbs / peak, 4),
                                        "share": 1.0},
                   "separate_calls": kernels}
        dom = "fused_moe_kernel"
    traffic = recorded_traffic(dom, wl.name)
    tokens = T * K * world
    value = job_rate(T * K, world, total_ms)
    # per layer: router (+ top-k and union kernels above 8 tokens), gate/up, down, the
    # stack's RMSNorm, and the layer call's x digit-record launch for up to 8 tokens
    launches_per_step = NL * ((1 if T <= 8 else 3) + 2 + (1 if stack else 0)
                              + (1 if args.api == "layer" and T <= 8 else 0))
    if fused:
        launches_per_step = 1 if stack else NL

    out = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": K,
        "warmup": args.warmup,
        "ms_per_step": round(total_ms / K, 6),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f32",
        "data": "synthetic",
        "config": workload_config(wl),
        "method": {"l2": "flushed before every step (2x L2 write, then 2x L2 read of another buffer), outside the timed intervals",
                   "timing": "CUDA graphs of up to 128 steps; events around each step (the value); "
                             "per-kernel figures from a second pass with events around each launch "
                             "(separate route_union / gate_up / down calls)",
                   "api": (("coli_moe_stack, one call (one launch) per step" if stack and fused else
                            "coli_moe_layer, one call per layer" + (" (one fused launch)" if fused else ""))
                           if args.api == "layer"
                           else "coli_moe_route_union + coli_moe_gate_up + coli_moe_down"),
                   "token_pool": R, "parallelism": f"replicas x{world}",
                   "mean_union_per_layer": float(nu.mean() / NL)},
        "roofline": {"bound": "hbm", "kernel": dom, "achieved": kernels[dom]["gb_s"],
                     "peak": peak, "peak_kind": f"{peak_kind} copy bandwidth",
                     "unit": "GB/s", "frac": kernels[dom]["frac"],
                     "traffic": traffic},
        "step_hbm": {"algorithmic_bytes": float(step_bytes.mean()),
                     "gb_s": round(float(step_bytes.sum() / (total_ms * 1e-3) / 1e9 * world), 1),
                     "frac_of_peak_per_gpu": round(float(step_bytes.sum() / (total_ms * 1e-3) / 1e9 / peak), 4)},
        "kernels": kernels,
        "gpu_launches": launches_per_step * K,
        "clocks": clocks,
    }
    if e2e:
        out["e2e"] = {"value": round(tokens / (e2e_ms * 1e-3), 2), "unit": "tokens/s",
                      "h2d_bytes_per_step": e2e[1], "d2h_bytes_per_step": e2e[2],
                      "api": "coli_moe_layer with pinned-host x in and y out"}
    if stack:
        out["method"]["kernel_figures"] = ("the step is one launch" if fused else
                                           f"per step (sum over the {NL} layers' launches)")
    if e2e and stack and fused:
        out["e2e"]["api"] = "coli_moe_stack with pinned-host x in and y out"
    if args.steady and not stack and fused:
        out["steady_state"] = steady_state(args, B, dims, layers[0], s, xs, bufs, float(step_bytes.mean()), l2,
                                           dev, peak)
    if world == 1 and not args.no_cpu_baseline and not stack:
        out["cpu_baseline"] = cpu_baseline(wl, args.cpu_seconds)
    return out


def steady_state(args, B, dims, L0, s, xs, bufs, call_bytes, l2, dev, peak):
    """Back-to-back fused layer calls with no flush between them, each reading a different
    copy of the layer's weights, the copies together at least 3x L2 of what the calls read,
    so every call streams its experts from HBM while the calls follow each other as in a
    decode loop."""
    import math

    import torch
    C = max(2, math.ceil(3 * l2 / max(call_bytes, 1.0)))
    copies = []
    for c in range(C):
        ex = L0["experts"].clone()
        sh = L0["shared"].clone()
        copies.append((ex, sh, B.make_weights(L0["wr"], L0["bias"], ex, sh, s.stride)))
    T, R = xs[0].shape[0], len(xs)
    n = 256

    def call(i):
        B.check(B.coli_moe_layer(dims, copies[i % C][2], xs[i % R], T, bufs.idx, bufs.w, None,
                                 bufs.union_ids, bufs.n_union, bufs.offsets, bufs.assign, None, bufs.y,
                                 bufs.ws), "coli_moe_layer")
    for i in range(2 * C):
        call(i)
    torch.cuda.synchronize(dev)
    ev = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(2)]
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        ev[0].record()
        for i in range(n):
            call(i)
        ev[1].record()
    g.replay()
    torch.cuda.synchronize(dev)
    best = None
    for _ in range(3):
        g.replay()
        torch.cuda.synchronize(dev)
        ms = ev[0].elapsed_time(ev[1])
        best = ms if best is None or ms < best else best
    del g
    per = best / n
    gbs = call_bytes / (per * 1e-3) / 1e9
    return {"ms_per_call": round(per, 6), "value": round(T / (per * 1e-3), 2), "unit": "tokens/s",
            "gb_s": round(gbs, 1), "frac": round(gbs / peak, 4), "weight_copies": C,
            "calls": n, "timing": "one CUDA graph of back-to-back calls, events at its two ends, "
                                  "best of 3 replays; no L2 flush (each call reads another copy)"}


def measured_tflops():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["bf16_tflops"]), float(d["bf16_tflops_sustained"]), "measured"
    return 1590.0, 1400.0, "fallback"


def run_prefill(args, wl, rank, world, dev):
    """Large bf16 batches: route + union, then the grouped tensor-core forward."""
    import torch

    from int4_routed_expert_gemv_b200 import binding as B
    from int4_routed_expert_gemv_b200 import synth

    s = wl.shape
    T = wl.tokens
    H, I, E, k = s.hidden, s.inter, s.n_experts, s.top_k
    ex = synth.experts_tensor(s, wl.seed, 0, device=dev)
    sh = synth.shared_tensor(s, wl.seed, 0, device=dev)
    wr = torch.from_numpy(synth.router_weight(s, wl.seed)).to(dev)
    bias = torch.from_numpy(synth.zipf_bias(E)).to(dev) if wl.zipf else None
    dims = B.make_dims(H, I, E, k, s.n_shared)
    weights = B.make_weights(wr, bias, ex, sh, s.stride)
    bufs = B.LayerBuffers(dims, T, device=dev)
    R = min(args.pool, 4)
    xs_host = [synth.activations_bf16(s, wl.seed, T, wl.x_variant + 100 * i).pin_memory()
               for i in range(R)]
    xs = [x.to(dev) for x in xs_host]
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    flush_buf = torch.empty(2 * l2 // 4 + 1024, dtype=torch.float32, device=dev)
    flush_read = torch.zeros(2 * l2 // 4 + 1024, dtype=torch.float32, device=dev)
    flush_sink = torch.empty(1, dtype=torch.float32, device=dev)
    y_host = torch.empty(T, H, dtype=torch.float32).pin_memory()

    def flush():
        flush_buf.zero_()
        torch.sum(flush_read, dim=0, keepdim=True, out=flush_sink)

    def step(i, ev=None):
        x = xs[i % R]
        if ev:
            ev[0].record()
        B.check(B.coli_moe_route_union(dims, wr, bias, x, T, bufs.idx, bufs.w, None, bufs.union_ids,
                                       bufs.n_union, bufs.offsets, bufs.assign, bufs.ws), "route")
        if ev:
            ev[1].record()
        B.check(B.coli_moe_forward(dims, weights, x, T, bufs.idx, bufs.w, bufs.union_ids,
                                   bufs.n_union, bufs.offsets, bufs.assign, None, bufs.y, bufs.ws),
                "forward")
        if ev:
            ev[2].record()

    # useful work per batch: union sizes and routed token counts
    for i in range(R):
        step(i)
    torch.cuda.synchronize(dev)
    gpu_id = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    sampler = ClockSampler(gpu_id)
    sampler.start()
    time.sleep(0.2)
    for i in range(args.warmup):
        flush()
        step(i)
    torch.cuda.synchronize(dev)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    K = args.steps
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
    t0 = time.time()
    for i in range(K):
        flush()
        step(args.warmup + i, evs[i])
    torch.cuda.synchronize(dev)
    t1 = time.time()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    time.sleep(0.1)
    sampler.stop()
    clocks = sampler.summary(t0, t1)
    seg = np.array([[evs[i][j].elapsed_time(evs[i][j + 1]) for j in range(2)] for i in range(K)])
    total_ms = float(seg.sum())
    st, bits = B.coli_moe_read_status(bufs.ws)
    if st != B.COLI_OK:
        raise SystemExit(f"device status {bits:#x} after the timed region")
    # e2e: host x in, y out, through coli_moe_layer
    e2e_ms = None
    if not args.no_e2e:
        ev2 = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
        xin = torch.empty_like(xs[0])
        for i in range(K):
            flush()
            ev2[i][0].record()
            xin.copy_(xs_host[i % R], non_blocking=True)
            B.check(B.coli_moe_layer(dims, weights, xin, T, bufs.idx, bufs.w, None, bufs.union_ids,
                                     bufs.n_union, bufs.offsets, bufs.assign, None, bufs.y, bufs.ws))
            y_host.copy_(bufs.y[:T], non_blocking=True)
            ev2[i][1].record()
        torch.cuda.synchronize(dev)
        e2e_ms = float(sum(ev2[i][0].elapsed_time(ev2[i][1]) for i in range(K)))
    total_ms, e2e_ms2 = max_over_ranks([total_ms, e2e_ms or 0.0], world, dev)
    if rank != 0:
        return None
    flops = 2.0 * 3.0 * H * I * T * (k + s.n_shared)          # useful: every routed token + shared
    burst, sustained, kind = measured_tflops()
    fwd_ms = seg[:, 1]
    tflops = flops / (fwd_ms.mean() * 1e-3) / 1e12
    tokens = T * K * world
    out = {
        "metric": "MoE-layer tokens/s; grouped-GEMM bf16 TFLOP/s as fraction of B200 dense peak (prefill)",
        "value": round(job_rate(T * K, world, total_ms), 1),
        "unit": "tokens/s",
        "n_gpus": world, "steps": K, "warmup": args.warmup,
        "ms_per_step": round(total_ms / K, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": workload_config(wl),
        "method": {"weights": "gs64 int4, fp16 scales, dequantised to bf16",
                   "l2": "flushed before every step, outside the timed intervals",
                   "parallelism": f"replicas x{world}", "n_union": int(bufs.n_union[0].item())},
        "roofline": {"bound": "tensor", "kernel": "grouped forward (gather + plan + 2 tcgen05 GEMM launches)",
                     "achieved": round(tflops, 1), "peak": burst,
                     "peak_kind": f"{kind} cuBLAS bf16 burst", "unit": "TFLOP/s",
                     "frac": round(tflops / burst, 4), "frac_of_sustained": round(tflops / sustained, 4),
                     "useful_flops_per_launch": flops, "traffic": None},
        "kernels": {"route_union": {"avg_us": round(float(seg[:, 0].mean()) * 1e3, 2)},
                    "forward": {"avg_us": round(float(fwd_ms.mean()) * 1e3, 2)}},
        "gpu_launches": K * (3 + 4),
        "clocks": clocks,
    }
    if e2e_ms is not None:
        out["e2e"] = {"value": round(tokens / (e2e_ms2 * 1e-3), 1), "unit": "tokens/s",
                      "h2d_bytes_per_step": T * H * 2, "d2h_bytes_per_step": T * H * 4,
                      "api": "coli_moe_layer with pinned-host x in and y out"}
    return out


# ------------------------------------------------------------------------------------
# the oracle on the host cores (CPU baseline and the reference arm)
# ------------------------------------------------------------------------------------

def oracle_setup(wl, n_batches):
    import oracle
    from int4_routed_expert_gemv_b200 import synth
    s = wl.shape
    wr = synth.router_weight(s, wl.seed)
    bias = synth.zipf_bias(s.n_experts) if wl.zipf else None
    batches = []
    blobs = {}
    for i in range(n_batches):
        x = synth.activations(s, wl.seed, wl.tokens, 1000 + i)
        idx, _, _ = oracle.route(x, wr, bias, s.top_k)
        for e in np.unique(idx):
            if int(e) not in blobs:
                blobs[int(e)] = synth.expert_blob(s, wl.seed, 0, int(e)).numpy()
        batches.append(x)
    shared = synth.expert_blob(s, wl.seed, 0, s.n_experts).numpy()
    return wr, bias, batches, blobs, shared


def oracle_step(wl, wr, bias, x, blobs, shared):
    import oracle
    s = wl.shape
    idx, w, _ = oracle.route(x, wr, bias, s.top_k)
    oracle.union(idx, s.n_experts)
    sub = {int(e): blobs[int(e)] for e in np.unique(idx)}
    return oracle.forward_sparse(s.hidden, s.inter, s.top_k, s.n_shared, x, sub, shared, idx, w)


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


def oracle_rate(wl, seconds, threads, setup):
    """Steps of the oracle done by `threads` threads in about `seconds` (the scalar C
    oracle runs without the interpreter lock, so the threads run in parallel); every
    thread finishes the step it is in."""
    import threading
    wr, bias, batches, blobs, shared = setup
    counts = [0] * threads
    deadline = time.perf_counter() + seconds

    def work(j):
        n = 0
        while True:
            oracle_step(wl, wr, bias, batches[(j + n) % len(batches)], blobs, shared)
            n += 1
            if time.perf_counter() >= deadline or n >= 64:
                break
        counts[j] = n

    t0 = time.perf_counter()
    ts = [threading.Thread(target=work, args=(j,)) for j in range(threads)]
    for t in ts:
        t.start()
    for t in ts:
        t.join()
    el = time.perf_counter() - t0
    return sum(counts), el


def cpu_baseline(wl, seconds):
    setup = oracle_setup(wl, 4)
    n1, el1 = oracle_rate(wl, seconds / 3, 1, setup)
    nth = os.cpu_count() or 1
    nn, eln = oracle_rate(wl, 2 * seconds / 3, nth, setup)
    return {"value": round(nn * wl.tokens / eln, 4), "unit": "tokens/s", "cores": nth,
            "kind": "oracle", "cpu_model": cpu_model(),
            "sample": f"{nn} steps of {wl.tokens} token(s) of {wl.name} on {nth} threads in {eln:.1f} s "
                      "(route+union+forward, scalar C, double accumulation, one step per thread at a time)",
            "one_thread": {"value": round(n1 * wl.tokens / el1, 4), "unit": "tokens/s", "cores": 1,
                           "sample": f"{n1} steps in {el1:.1f} s"}}


def workload_config(wl):
    """The `config` object of a workload (shared by both arms)."""
    s = wl.shape
    return {"workload": wl.name, "tokens_per_step": wl.tokens, "layers": wl.layers, "hidden": s.hidden,
            "intermediate": s.inter, "experts": s.n_experts, "top_k": s.top_k,
            "shared_experts": s.n_shared, "weights": "gs64 int4, fp16 scales",
            "activations": "bf16" if wl.x_dtype == "bf16" else "fp32"}


def run_reference(args, rank):
    if rank != 0:
        return None
    from int4_routed_expert_gemv_b200 import synth
    import oracle
    oracle.build()
    wl = synth.WORKLOADS[args.workload]
    wr, bias, batches, blobs, shared = oracle_setup(wl, 4)
    # the oracle is a plain scalar C loop (seconds per GLM-shaped step): at most one untimed
    # step, then timed steps until --ref-seconds have passed (at least one), so any
    # --steps/--warmup finishes in about a minute; the rate is steps done / time taken
    for i in range(min(args.warmup, 1)):
        oracle_step(wl, wr, bias, batches[i % 4], blobs, shared)
    t0 = time.perf_counter()
    done = 0
    while done < args.steps:
        oracle_step(wl, wr, bias, batches[done % 4], blobs, shared)
        done += 1
        if time.perf_counter() - t0 > args.ref_seconds:
            break
    el = time.perf_counter() - t0
    v = done * wl.tokens / el
    return {"impl": "reference", "metric": METRIC, "value": round(v, 4), "unit": "tokens/s",
            "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(el * 1e3 / done, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(wl),
            "cpu_baseline": {"value": round(v, 4), "unit": "tokens/s", "cores": 1,
                             "kind": "oracle",
                             "sample": f"{done} timed step(s) of {wl.tokens} token(s) "
                                       f"(of {args.steps} requested; time-bounded at {args.ref_seconds:g} s), "
                                       "rotating over 4 token batches"},
            "e2e": {"value": round(v, 4), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


# The other configurations, each run by a short bench of its own (a subprocess, so that
# each holds only its own weights): (workload, steps, extra flags)
OTHER_CONFIGS = [
    ("moe_h1024_i512_e64_k4_t1", 200, ["--steady"]),
    ("moe_h1024_i512_e64_k4_t4_zipf", 200, ["--steady"]),
    ("glm52_moe_h6144_i2048_e256_k8_t4_zipf", 100, []),
    ("moe_h1024_i512_e64_k4_stack16_t1", 50, []),
    ("glm52_stack16_h6144_i2048_e256_k8_t1", 20, []),
    ("moe_h1024_i512_e64_k4_t2048_bf16_zipf", 20, []),
    ("glm52_moe_h6144_i2048_e256_k8_t2048_bf16_zipf", 10, []),
]


def run_formats(args):
    """The weight containers side by side.  Speed: the GLM-shaped layer (hidden 6144, 256
    experts, top-8 + shared), one token, random payloads, coli_moe_forward_fmt timed in
    CUDA graphs with an L2 flush before every call.  Accuracy: the hidden-1024 layer with
    fp32 weights N(0, 0.05) quantised by the package's host quantiser, y of the GPU path
    against the same layer with the unquantised weights (numpy, double)."""
    import torch

    from int4_routed_expert_gemv_b200 import binding as B
    from int4_routed_expert_gemv_b200 import build as builder
    from int4_routed_expert_gemv_b200 import quantize as Q
    from int4_routed_expert_gemv_b200 import synth
    builder.build()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    names = {0: "int4_gs64", 1: "int8_gs64", 2: "int4_per_row", 3: "int2_gs64"}
    peak, peak_kind = measured_peaks()
    out = {}
    # speed at the GLM shape
    s = synth.GLM
    H, I, E, k = s.hidden, s.inter, s.n_experts, s.top_k
    dims = B.make_dims(H, I, E, k, 1)
    wr = torch.from_numpy(synth.router_weight(s, 1)).to(dev)
    R = 16
    xs = [torch.from_numpy(synth.activations(s, 1, 1, 2000 + i)).to(dev) for i in range(R)]
    routes = []
    for i in range(R):
        b = B.LayerBuffers(dims, 1, device=dev)
        B.check(B.coli_moe_route_union(dims, wr, None, xs[i], 1, b.idx, b.w, None, b.union_ids, b.n_union,
                                       b.offsets, b.assign, b.ws))
        routes.append(b)
    torch.cuda.synchronize(dev)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    flush_buf = torch.empty(2 * l2 // 4 + 1024, dtype=torch.float32, device=dev)
    y = torch.empty(1, H, device=dev)
    K = min(args.steps, 100)
    for fmt in range(4):
        bb = B.coli_moe_blob_bytes_fmt(H, I, fmt)
        stride = (bb + 255) // 256 * 256
        qb = 3 * H * I * Q.BITS[fmt] // 8
        ex = torch.randint(0, 256, (E + 1, stride), dtype=torch.uint8, device=dev)
        ex[:, qb:bb].view(torch.float16).fill_(0.01)
        wts = B.make_weights(wr, None, ex[:E].reshape(-1), ex[E], stride)
        def call(i):
            b = routes[i % R]
            B.check(B.coli_moe_forward_fmt(dims, fmt, wts, xs[i % R], 1, b.w, b.union_ids, b.n_union, b.offsets,
                                           b.assign, None, y, b.ws))
        for i in range(3):
            call(i)
        torch.cuda.synchronize(dev)
        evs = [[torch.cuda.Event(enable_timing=True, external=True) for _ in range(2)] for _ in range(K)]
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for i in range(K):
                flush_buf.zero_()
                evs[i][0].record()
                call(i)
                evs[i][1].record()
        g.replay()
        torch.cuda.synchronize(dev)
        ms = float(np.mean([e[0].elapsed_time(e[1]) for e in evs]))
        del g
        nb = float(np.mean([int(routes[i % R].n_union[0].item()) for i in range(K)]))
        step_bytes = (nb + 1) * bb + E * H * 0
        gbs = step_bytes / (ms * 1e-3) / 1e9
        out[names[fmt]] = {"blob_bytes_glm": bb, "bits_per_weight": round(8.0 * bb / (3 * H * I), 4),
                           "glm_t1": {"us_per_call": round(ms * 1e3, 2), "expert_bytes": step_bytes,
                                      "gb_s": round(gbs, 1), "frac": round(gbs / peak, 4)}}
        del ex
    # accuracy at hidden 1024 against fp32 weights
    s1 = synth.LayerShape(1024, 512, 64, 4, 1)
    H1, I1, E1, k1 = s1.hidden, s1.inter, s1.n_experts, s1.top_k
    rng = np.random.default_rng(12)
    Wf = [[(rng.standard_normal(shp) * 0.05).astype(np.float32) for shp in ((I1, H1), (I1, H1), (H1, I1))]
          for _ in range(E1 + 1)]
    dims1 = B.make_dims(H1, I1, E1, k1, 1)
    wr1_h = synth.router_weight(s1, 0)
    wr1 = torch.from_numpy(wr1_h).to(dev)
    T1 = 4
    x1_h = synth.activations(s1, 0, T1, 300)
    x1 = torch.from_numpy(x1_h).to(dev)
    b1 = B.LayerBuffers(dims1, T1, device=dev)
    B.check(B.coli_moe_route_union(dims1, wr1, None, x1, T1, b1.idx, b1.w, None, b1.union_ids, b1.n_union,
                                   b1.offsets, b1.assign, b1.ws))
    idx = b1.idx[:T1].cpu().numpy()
    wgt = b1.w[:T1].cpu().numpy().astype(np.float64)

    def expert64(G, U, D, xt):
        g = G.astype(np.float64) @ xt
        u = U.astype(np.float64) @ xt
        return D.astype(np.float64) @ (g / (1.0 + np.exp(-g)) * u)
    y32 = np.zeros((T1, H1))
    for t in range(T1):
        xt = x1_h[t].astype(np.float64)
        y32[t] = expert64(*Wf[E1], xt) + sum(wgt[t, j] * expert64(*Wf[idx[t, j]], xt) for j in range(k1))
    for fmt in range(4):
        bb = B.coli_moe_blob_bytes_fmt(H1, I1, fmt)
        stride = (bb + 255) // 256 * 256
        host = np.zeros((E1 + 1, stride), np.uint8)
        for e in range(E1 + 1):
            host[e, :bb] = Q.expert_blob(*Wf[e], fmt)[0]
        ex = torch.from_numpy(host).to(dev)
        wts = B.make_weights(wr1, None, ex[:E1].reshape(-1), ex[E1], stride)
        y1 = torch.empty(T1, H1, device=dev)
        B.check(B.coli_moe_forward_fmt(dims1, fmt, wts, x1, T1, b1.w, b1.union_ids, b1.n_union, b1.offsets,
                                       b1.assign, None, y1, b1.ws))
        yq = y1.cpu().numpy().astype(np.float64)
        out[names[fmt]]["h1024_t4_rel_l2_vs_fp32_weights"] = float(
            np.linalg.norm(yq - y32) / np.linalg.norm(y32))
    return {"formats": out, "peak": peak, "peak_kind": f"{peak_kind} copy bandwidth",
            "method": "speed: coli_moe_forward_fmt (two launches), GLM shape, T=1, random payloads, "
                      f"CUDA graph of {K} calls with an L2 flush before each; accuracy: hidden 1024, T=4, "
                      "fp32 weights N(0, 0.05) quantised by quantize.py, vs the fp32-weight layer in double"}


def run_other_configs(args):
    import subprocess
    res = {}
    for name, steps, extra in OTHER_CONFIGS:
        cmd = [sys.executable, os.path.abspath(__file__), "--workload", name, "--steps", str(steps),
               "--warmup", "3", "--no-cpu-baseline", "--no-e2e", "--no-configs"] + extra
        try:
            p = subprocess.run(cmd, capture_output=True, text=True, timeout=300)
            line = [l for l in p.stdout.splitlines() if l.startswith("{")]
            if p.returncode != 0 or not line:
                res[name] = {"error": (p.stderr.strip().splitlines() or ["no output"])[-1][:300]}
                continue
            o = json.loads(line[-1])
        except subprocess.TimeoutExpired:
            res[name] = {"error": "timed out after 300 s"}
            continue
        r = {"value": o["value"], "unit": o["unit"], "ms_per_step": o["ms_per_step"], "steps": o["steps"],
             "roofline": o.get("roofline"), "clocks": o.get("clocks")}
        for key in ("step_hbm", "steady_state", "method"):
            if key in o:
                r[key] = o[key]
        res[name] = r
    # the weight containers (a bench of their own)
    cmd = [sys.executable, os.path.abspath(__file__), "--formats-only", "--steps", "100"]
    try:
        p = subprocess.run(cmd, capture_output=True, text=True, timeout=300)
        line = [l for l in p.stdout.splitlines() if l.startswith("{")]
        res["weight_containers"] = json.loads(line[-1]) if p.returncode == 0 and line else \
            {"error": (p.stderr.strip().splitlines() or ["no output"])[-1][:300]}
    except subprocess.TimeoutExpired:
        res["weight_containers"] = {"error": "timed out after 300 s"}
    return res


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        out = run_reference(args, rank)
        if out is not None:
            print(json.dumps(out), flush=True)
        return
    if args.formats_only:
        print(json.dumps(run_formats(args)), flush=True)
        return
    if world > 1:
        import datetime

        import torch
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                             device_id=torch.device("cuda", local_rank))
    try:
        out = run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch
            torch.distributed.destroy_process_group()
    if out is not None and world == 1 and not args.no_configs and args.workload == DEFAULT_WORKLOAD:
        import torch
        torch.cuda.empty_cache()
        out["configs"] = run_other_configs(args)
    if out is not None:
        print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()
