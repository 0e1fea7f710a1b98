"""Test helpers: seeded layers on the device and the oracle-side view of the same layer.

Inputs come only from the seeded generators; expected values come only from the oracle.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, Optional

import numpy as np
import torch

import oracle
from int4_routed_expert_gemv_b200 import binding as B
from int4_routed_expert_gemv_b200 import synth

# parity bars for floating-point outputs
Y_REL_L2 = 1e-4          # ||y - y_oracle|| / ||y_oracle||
Y_MAX_ABS_RMS = 1e-3     # max |y - y_oracle| / rms(y_oracle)
W_ABS = 1e-6             # routing weights


@dataclasses.dataclass
class DeviceLayer:
    shape: synth.LayerShape
    seed: int
    layer: int
    experts: torch.Tensor          # [E][stride] uint8, device
    shared: Optional[torch.Tensor]
    w_router: torch.Tensor         # [E][H] fp32, device
    bias: Optional[torch.Tensor]
    w_router_host: np.ndarray
    bias_host: Optional[np.ndarray]
    dims: B.Dims = None
    weights: B.Weights = None

    def blob_host(self, e: int) -> np.ndarray:
        """Expert e's blob regenerated on the host (e == E: shared expert)."""
        return synth.expert_blob(self.shape, self.seed, self.layer, e, device="cpu").numpy()

    def all_blobs_host(self) -> np.ndarray:
        return synth.experts_tensor(self.shape, self.seed, self.layer, device="cpu").numpy()


def make_device_layer(shape: synth.LayerShape, seed: int, layer: int = 0, zipf: bool = False,
                      device="cuda", w_router_host: Optional[np.ndarray] = None,
                      bias_host: Optional[np.ndarray] = None) -> DeviceLayer:
    experts = synth.experts_tensor(shape, seed, layer, device=device)
    shared = synth.shared_tensor(shape, seed, layer, device=device) if shape.n_shared else None
    wr = synth.router_weight(shape, seed, layer) if w_router_host is None else w_router_host
    if bias_host is None and zipf:
        bias_host = synth.zipf_bias(shape.n_experts)
    L = DeviceLayer(shape, seed, layer, experts, shared,
                    torch.from_numpy(np.ascontiguousarray(wr)).to(device),
                    None if bias_host is None else torch.from_numpy(bias_host).to(device),
                    wr, bias_host)
    L.dims = B.make_dims(shape.hidden, shape.inter, shape.n_experts, shape.top_k, shape.n_shared)
    L.weights = B.make_weights(L.w_router, L.bias, L.experts, L.shared, shape.stride)
    return L


def oracle_layer(L: DeviceLayer, x: np.ndarray, bf16: bool = False,
                 blobs: Optional[Dict[int, np.ndarray]] = None) -> dict:
    """Oracle route -> union -> forward for x [T][H] (float32 values)."""
    s = L.shape
    idx, w, logits = oracle.route(x, L.w_router_host, L.bias_host, s.top_k)
    uid, nu, off, asg = oracle.union(idx, s.n_experts)
    if blobs is None:
        blobs = {int(e): L.blob_host(int(e)) for e in np.unique(idx)}
    shared = L.blob_host(s.n_experts) if s.n_shared else None
    y = oracle.forward_sparse(s.hidden, s.inter, s.top_k, s.n_shared, x, blobs, shared, idx, w,
                              bf16=bf16)
    return dict(idx=idx, w=w, logits=logits, union_ids=uid, n_union=nu, offsets=off, assign=asg,
                y=y)


def y_errors(y: np.ndarray, ref: np.ndarray):
    y = y.astype(np.float64)
    ref = ref.astype(np.float64)
    d = y - ref
    rms = float(np.sqrt(np.mean(ref ** 2))) if ref.size else 0.0
    rel = float(np.linalg.norm(d) / max(np.linalg.norm(ref), 1e-300))
    mx = float(np.abs(d).max() / max(rms, 1e-300)) if ref.size else 0.0
    return rel, mx


def assert_y_close(y: np.ndarray, ref: np.ndarray, rel_l2=Y_REL_L2, max_rms=Y_MAX_ABS_RMS):
    rel, mx = y_errors(y, ref)
    assert rel <= rel_l2 and mx <= max_rms, f"rel L2 {rel:.3e} (bar {rel_l2}), " \
                                            f"max/rms {mx:.3e} (bar {max_rms})"
    return rel, mx


def run_layer(L: DeviceLayer, x_dev: torch.Tensor, T: int, residual=None, bufs=None):
    """One fused coli_moe_layer call; returns host copies of every output."""
    bufs = bufs or B.LayerBuffers(L.dims, T)
    B.check(B.coli_moe_layer(L.dims, L.weights, x_dev, T, bufs.idx, bufs.w, bufs.logits,
                             bufs.union_ids, bufs.n_union, bufs.offsets, bufs.assign, residual,
                             bufs.y, bufs.ws), "coli_moe_layer")
    st, bits = B.coli_moe_read_status(bufs.ws)
    assert st == B.COLI_OK and bits == 0, f"device status {bits:#x}"
    return host_outputs(bufs, T, L.shape)


def host_outputs(bufs, T, shape):
    k, E = shape.top_k, shape.n_experts
    return dict(idx=bufs.idx[:T].cpu().numpy(), w=bufs.w[:T].cpu().numpy(),
                logits=bufs.logits[:T].cpu().numpy(), union_ids=bufs.union_ids.cpu().numpy(),
                n_union=int(bufs.n_union[0].item()), offsets=bufs.offsets.cpu().numpy(),
                assign=bufs.assign[:T * k].cpu().numpy(), y=bufs.y[:T].cpu().numpy())


def assert_route_union_equal(got: dict, ref: dict, check_logits=True):
    assert np.array_equal(got["idx"], ref["idx"]), "expert indices differ"
    assert np.abs(got["w"] - ref["w"]).max() <= W_ABS
    if check_logits:
        assert np.array_equal(got["logits"], ref["logits"]), "logits differ"
    assert got["n_union"] == ref["n_union"]
    assert np.array_equal(got["union_ids"], ref["union_ids"])
    assert np.array_equal(got["offsets"], ref["offsets"])
    assert np.array_equal(got["assign"], ref["assign"])
