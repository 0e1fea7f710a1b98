"""The grouped tensor-core path (bf16 activations, bf16 contract) against the oracle's
bf16-weights mode: every weight bf16(q * scale), x bf16 as given, h exact, sums in double
(the device carries h into the down projection as a bf16 hi + lo pair).

Routing, union and assignment lists are checked bit for bit for every token.  y, within
relative L2 1e-4 and max 1e-3 rms: at hidden 1024 on every token; at the GLM shape (the
scalar oracle costs ~0.5 s per token) on the first and last token of three experts of
every group-size class (up to 16, 32, 64, 128 tokens and more, the token-box heights
of the grouped GEMM), plus the batch's first and last token.
"""
import numpy as np
import pytest
import torch

import oracle
from int4_routed_expert_gemv_b200 import binding as B
from int4_routed_expert_gemv_b200 import synth
from layers import assert_route_union_equal, assert_y_close, host_outputs, make_device_layer

pytestmark = pytest.mark.gpu


def run_bf16(L, x_bf16: torch.Tensor, T, residual=None):
    bufs = B.LayerBuffers(L.dims, T)
    B.check(B.coli_moe_layer(L.dims, L.weights, x_bf16.cuda(), T, bufs.idx, bufs.w, bufs.logits,
                             bufs.union_ids, bufs.n_union, bufs.offsets, bufs.assign, residual,
                             bufs.y, bufs.ws), "coli_moe_layer(bf16)")
    st, bits = B.coli_moe_read_status(bufs.ws)
    assert st == B.COLI_OK and bits == 0, f"device status {bits:#x}"
    return host_outputs(bufs, T, L.shape)


def check_layer(L, x_bf16, T, sample, residual=None):
    x32 = x_bf16.float().numpy()
    got = run_bf16(L, x_bf16, T, None if residual is None else torch.from_numpy(residual).cuda())
    s = L.shape
    idx, w, logits = oracle.route(x32, L.w_router_host, L.bias_host, s.top_k)
    uid, nu, off, asg = oracle.union(idx, s.n_experts)
    ref = dict(idx=idx, w=w, logits=logits, union_ids=uid, n_union=nu, offsets=off, assign=asg)
    assert_route_union_equal(got, ref)
    rows = np.array(sorted(set(sample)), dtype=np.int64)
    blobs = {int(e): L.blob_host(int(e)) for e in np.unique(idx[rows])}
    shared = L.blob_host(s.n_experts) if s.n_shared else None
    y_ref = oracle.forward_sparse(s.hidden, s.inter, s.top_k, s.n_shared, x32[rows], blobs, shared,
                                  idx[rows], w[rows], bf16=2)
    y = got["y"][rows]
    if residual is not None:
        y = y - residual[rows]
    return assert_y_close(y, y_ref)


def group_edge_tokens(L, x_bf16, T):
    """First and last token of three experts (lowest, middle, highest id) in every class
    of token-group size, and the batch's first and last token."""
    s = L.shape
    idx, _, _ = oracle.route(x_bf16.float().numpy(), L.w_router_host, L.bias_host, s.top_k)
    uid, nu, off, asg = oracle.union(idx, s.n_experts)
    classes = {}
    for u in range(nu):
        c = off[u + 1] - off[u]
        b = 0 if c <= 16 else 1 if c <= 32 else 2 if c <= 64 else 3 if c <= 128 else 4
        classes.setdefault(b, []).append(u)
    tokens = {0, T - 1}
    for us in classes.values():
        for u in {us[0], us[len(us) // 2], us[-1]}:
            tokens.add(int(asg[off[u]]) // s.top_k)
            tokens.add(int(asg[off[u + 1] - 1]) // s.top_k)
    return sorted(tokens)


@pytest.mark.parametrize("name", ["moe_h1024_i512_e64_k4_t2048_bf16_zipf",
                                  "glm52_moe_h6144_i2048_e256_k8_t2048_bf16_zipf"])
def test_prefill_grouped_gemm(colimoe, name):
    wl = synth.WORKLOADS[name]
    L = make_device_layer(wl.shape, wl.seed, zipf=wl.zipf)
    x = synth.activations_bf16(wl.shape, wl.seed, wl.tokens, wl.x_variant)
    if wl.shape.hidden <= 1024:
        sample = list(range(wl.tokens))
    else:
        sample = group_edge_tokens(L, x, wl.tokens)
    rel, mx = check_layer(L, x, wl.tokens, sample)
    print(f"{name}: rel L2 {rel:.2e}, max/rms {mx:.2e}")


@pytest.mark.parametrize("T", [1, 3, 37, 300])
@pytest.mark.parametrize("ns", [1, 0])
def test_small_and_ragged_bf16_batches(colimoe, T, ns):
    shape = synth.LayerShape(1024, 512, 64, 4, ns)
    L = make_device_layer(shape, 31 + T, zipf=True)
    x = synth.activations_bf16(shape, 31, T, 4)
    res = synth.activations(shape, 99, T, 1) if ns else None
    sample = list(range(min(T, 12))) + [T - 1]
    check_layer(L, x, T, sample, residual=res)
