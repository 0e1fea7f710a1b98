"""Phase timeline of the fused decode launch (one layer, 1-4 tokens).

    python -m int4_routed_expert_gemv_b200.phases [workload] [--reps 3]

Builds (if needed) and loads the phase-stamp build of the library (COLI_PHASE_STAMPS:
the same kernels with one global-timer store per CTA at each phase boundary), runs the
workload's layer with L2 flushed before every call, and prints, per phase, the minimum,
median and maximum over the CTAs of the time since the earliest CTA entered the kernel.
The stamps cost a few stores per CTA; the regular build has none.
"""
from __future__ import annotations

import argparse
import os

import numpy as np
import torch

PHASES = ["kernel entry", "layer input loaded", "router partials published", "input operand built",
          "routing table ready", "first routed gate/up stage", "first down stage",
          "last down stage done", "last reduction done", "exit"]


def main(argv=None):
    from . import build, synth
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("workload", nargs="?", default="glm52_moe_h6144_i2048_e256_k8_t1")
    ap.add_argument("--reps", type=int, default=3)
    a = ap.parse_args(argv)
    wl = synth.WORKLOADS[a.workload]
    if wl.layers != 1 or wl.tokens > 4 or wl.x_dtype != "f32":
        raise SystemExit("the phase timeline covers one-layer decode workloads (1-4 fp32 tokens)")
    from . import binding as B
    B.LIB_PATH = build.build(stamps=True)
    s, T = wl.shape, wl.tokens
    dims = B.make_dims(s.hidden, s.inter, s.n_experts, s.top_k, s.n_shared)
    experts = synth.experts_tensor(s, wl.seed, device="cuda")
    shared = synth.shared_tensor(s, wl.seed, device="cuda")
    wr = torch.from_numpy(synth.router_weight(s, wl.seed)).cuda()
    bias = torch.from_numpy(synth.zipf_bias(s.n_experts)).cuda() if wl.zipf else None
    weights = B.make_weights(wr, bias, experts.reshape(-1), shared, s.stride)
    x = torch.from_numpy(synth.activations(s, wl.seed, T, wl.x_variant)).cuda()
    bufs = B.LayerBuffers(dims, T)
    flush = torch.empty(512 << 20, dtype=torch.uint8, device="cuda")

    def run():
        B.check(B.coli_moe_layer(dims, weights, x, T, bufs.idx, bufs.w, None, bufs.union_ids, bufs.n_union,
                                 bufs.offsets, bufs.assign, None, bufs.y, bufs.ws), "coli_moe_layer")

    for _ in range(3):
        run()
    torch.cuda.synchronize()
    print(f"{a.workload}: phase times in us since the first CTA's entry (min / median / max over CTAs)")
    for rep in range(a.reps):
        flush.fill_(rep)
        torch.cuda.synchronize()
        run()
        torch.cuda.synchronize()
        st, tl = B.coli_debug_phase_stamps()
        B.check(st, "coli_debug_phase_stamps")
        if B.coli_moe_read_status(bufs.ws) != (B.COLI_OK, 0):
            raise SystemExit("device status set")
        tl = tl[tl[:, 0] > 0]            # the launch's CTAs
        t0 = tl[:, 0].min()
        print(f"--- call {rep}")
        for i, name in enumerate(PHASES):
            v = tl[:, i]
            v = (v[v > 0].astype(np.int64) - int(t0)) / 1000.0
            if len(v):
                print(f"  {name:28s} {v.min():8.2f} {np.median(v):8.2f} {v.max():8.2f}")


if __name__ == "__main__":
    main()
