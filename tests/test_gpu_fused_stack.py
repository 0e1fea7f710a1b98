"""The residual decode stack through coli_moe_stack: up to 16 layers in one launch, the
residual stream kept on the device (x <- x + MoE(RMSNorm(x)) per layer).

Checked against the oracle's layer chain (oracle.stack_layer, which regenerates only the
experts each layer selects):
  * teacher forcing: each layer run alone (n_layers = 1) from the oracle's input to that
    layer; its output minus its input must meet the per-layer float bar and select the same
    experts;
  * free running: all layers in one call select the same experts as the oracle at every
    layer and end within the float bar;
  * a stack longer than one launch (more than 16 layers) chains launches through the
    workspace and gives the same result as the layers run one by one.
"""
import numpy as np
import pytest
import torch

import oracle
from int4_routed_expert_gemv_b200 import binding as B
from int4_routed_expert_gemv_b200 import synth
from layers import assert_y_close, y_errors

pytestmark = pytest.mark.gpu


def _stack(wl, n_layers=None):
    s = wl.shape
    L = n_layers or wl.layers
    dims = B.make_dims(s.hidden, s.inter, s.n_experts, s.top_k, s.n_shared)
    layers = []
    for l in range(L):
        ex = synth.experts_tensor(s, wl.seed, l, device="cuda")
        sh = synth.shared_tensor(s, wl.seed, l, device="cuda")
        wr_h = synth.router_weight(s, wl.seed, l)
        wr = torch.from_numpy(wr_h).cuda()
        layers.append(dict(ex=ex, sh=sh, wr=wr, wr_h=wr_h, w=B.make_weights(wr, None, ex, sh, s.stride)))
    return dims, layers


def _oracle_chain(wl, layers, x0, gamma_h, eps=1e-5):
    s = wl.shape
    xs, idxs = [x0.copy()], []
    for l in range(len(layers)):
        get = lambda e, l=l: synth.expert_blob(s, wl.seed, l, e).numpy()
        shared = synth.expert_blob(s, wl.seed, l, s.n_experts).numpy()
        xn, nrm, idx, w, logits, y = oracle.stack_layer(xs[-1], gamma_h, eps, layers[l]["wr_h"], None,
                                                        s.top_k, s.hidden, s.inter, 1, get, shared)
        srt = np.sort(logits, axis=1)[:, ::-1]
        assert np.all(srt[:, s.top_k - 1] > srt[:, s.top_k]), f"layer {l}: exact tie at the boundary"
        xs.append(xn)
        idxs.append(idx)
    return xs, idxs


def _run_stack(dims, layers, gammas, x, T, n_idx, ws):
    y = torch.empty_like(x)
    idx = torch.full((n_idx, T, dims.top_k), -1, dtype=torch.int32, device="cuda")
    B.check(B.coli_moe_stack(dims, [l["w"] for l in layers], gammas, 1e-5, x, T, idx, y, ws),
            "coli_moe_stack")
    return y, idx


@pytest.mark.parametrize("T", [1, 2])
def test_h1024_stack16_teacher_forced_and_free_running(colimoe, T):
    wl = synth.WORKLOADS["moe_h1024_i512_e64_k4_stack16_t1"]
    s, L = wl.shape, wl.layers
    dims, layers = _stack(wl)
    gamma_h = np.ones(s.hidden, np.float32)
    gammas = [torch.from_numpy(gamma_h).cuda() for _ in range(L)]
    x0 = synth.activations(s, wl.seed, T, wl.x_variant)
    xs_o, idx_o = _oracle_chain(wl, layers, x0, gamma_h)
    ws = torch.zeros(B.coli_moe_workspace_bytes(dims, T), dtype=torch.uint8, device="cuda")
    B.check(B.coli_moe_workspace_init(ws))
    # teacher forcing, one layer per call
    for l in range(L):
        xl = torch.from_numpy(xs_o[l]).cuda()
        y, idx = _run_stack(dims, layers[l:l + 1], gammas[l:l + 1], xl, T, 1, ws)
        assert np.array_equal(idx[0].cpu().numpy(), idx_o[l]), f"layer {l}: experts differ"
        assert_y_close(y.cpu().numpy() - xs_o[l], xs_o[l + 1] - xs_o[l])
    # free running, all layers in one launch
    y, idx = _run_stack(dims, layers, gammas, torch.from_numpy(x0).cuda(), T, L, ws)
    for l in range(L):
        assert np.array_equal(idx[l].cpu().numpy(), idx_o[l]), f"free-running layer {l}: experts differ"
    rel, mx = y_errors(y.cpu().numpy(), xs_o[-1])
    print(f"T={T}: free-running 16-layer x rel L2 {rel:.2e} max/rms {mx:.2e}")
    assert_y_close(y.cpu().numpy(), xs_o[-1])
    st, bits = B.coli_moe_read_status(ws)
    assert st == B.COLI_OK and bits == 0


def test_stack_longer_than_one_launch(colimoe):
    # 20 layers (one launch of 16, one of 4) equal the same layers run one call each
    wl = synth.WORKLOADS["moe_h1024_i512_e64_k4_stack16_t1"]
    s = wl.shape
    dims, layers = _stack(wl, 20)
    T = 1
    x0 = torch.from_numpy(synth.activations(s, wl.seed, T, 5)).cuda()
    ws = torch.zeros(B.coli_moe_workspace_bytes(dims, T), dtype=torch.uint8, device="cuda")
    B.check(B.coli_moe_workspace_init(ws))
    y_all, idx_all = _run_stack(dims, layers, None, x0, T, 20, ws)
    x = x0
    for l in range(20):
        x, idx = _run_stack(dims, layers[l:l + 1], None, x, T, 1, ws)
        assert np.array_equal(idx[0].cpu().numpy(), idx_all[l].cpu().numpy())
    assert torch.equal(x, y_all), "a stack split over launches must equal the layers one by one"


def test_stack_rejects_bad_arguments(colimoe):
    wl = synth.WORKLOADS["moe_h1024_i512_e64_k4_stack16_t1"]
    dims, layers = _stack(wl, 2)
    x = torch.zeros(1, wl.shape.hidden, device="cuda")
    ws = torch.zeros(B.coli_moe_workspace_bytes(dims, 1), dtype=torch.uint8, device="cuda")
    B.check(B.coli_moe_workspace_init(ws))
    w = [l["w"] for l in layers]
    # y overlapping x
    assert B.coli_moe_stack(dims, w, None, 1e-5, x, 1, None, x, ws) == B.COLI_EINVAL
    # batches beyond the decode kernel
    y = torch.zeros(8, wl.shape.hidden, device="cuda")
    x8 = torch.zeros(8, wl.shape.hidden, device="cuda")
    ws8 = torch.zeros(B.coli_moe_workspace_bytes(dims, 8), dtype=torch.uint8, device="cuda")
    assert B.coli_moe_stack(dims, w, None, 1e-5, x8, 8, None, y, ws8) == B.COLI_EUNSUPPORTED
    # zero layers / zero tokens: no-op
    assert B.coli_moe_stack(dims, [], None, 1e-5, x, 1, None, y[:1], ws) == B.COLI_OK
