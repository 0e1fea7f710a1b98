"""16-layer residual decode stack of GLM-5.2-shaped MoE layers (82.6 GB of experts resident
in HBM): x <- x + MoE(RMSNorm(x)) per layer, one token, through the C ABI
(coli_rmsnorm + coli_moe_layer with the residual fused into the down projection).

The oracle runs the 16 layers on the host from the same seeded inputs, regenerating only
the experts each layer selects.  Checked:
  * teacher forcing: every layer of the GPU path is fed the oracle's input to that layer
    (oracle values into the device, never the reverse) and its output y_l = x_(l+1) - x_l
    must meet the per-layer float bar (relative L2 1e-4, max 1e-3 rms);
  * the free-running GPU stack selects the same experts as the oracle at every layer and
    ends within the same float bar.
"""
import numpy as np
import pytest
import torch

import oracle
from int4_routed_expert_gemv_b200 import binding as B
from int4_routed_expert_gemv_b200 import synth
from layers import assert_y_close, y_errors

pytestmark = pytest.mark.gpu


def test_glm_stack16_decode(colimoe):
    wl = synth.WORKLOADS["glm52_stack16_h6144_i2048_e256_k8_t1"]
    s, L, T = wl.shape, wl.layers, wl.tokens
    free, _ = torch.cuda.mem_get_info()
    need = L * (s.n_experts + 1) * s.stride
    assert free > need + (4 << 30), f"needs {need / 1e9:.1f} GB of free device memory"
    dims = B.make_dims(s.hidden, s.inter, s.n_experts, s.top_k, s.n_shared)
    layers = []
    for l in range(L):
        ex = synth.experts_tensor(s, wl.seed, l, device="cuda")
        sh = synth.shared_tensor(s, wl.seed, l, device="cuda")
        wr_h = synth.router_weight(s, wl.seed, l)
        wr = torch.from_numpy(wr_h).cuda()
        layers.append((ex, sh, wr, wr_h, B.make_weights(wr, None, ex, sh, s.stride)))
    gamma_h = np.ones(s.hidden, np.float32)
    gamma = torch.from_numpy(gamma_h).cuda()
    x0 = synth.activations(s, wl.seed, T, wl.x_variant)
    bufs = B.LayerBuffers(dims, T)

    def gpu_layer(l, x):
        n = torch.empty_like(x)
        B.check(B.coli_rmsnorm(s.hidden, T, x, gamma, 1e-5, n))
        B.check(B.coli_moe_layer(dims, layers[l][4], n, T, bufs.idx, bufs.w, None, bufs.union_ids,
                                 bufs.n_union, bufs.offsets, bufs.assign, x, x, bufs.ws))
        return bufs.idx[:T].cpu().numpy().copy()

    # oracle chain
    xs_o = [x0.copy()]
    idx_o = []
    for l in range(L):
        get = lambda e, l=l: synth.expert_blob(s, wl.seed, l, e).numpy()
        shared = synth.expert_blob(s, wl.seed, l, s.n_experts).numpy()
        xn, nrm, idx, w, logits, y = oracle.stack_layer(xs_o[-1], gamma_h, 1e-5, layers[l][3], None,
                                                        s.top_k, s.hidden, s.inter, 1, get, shared)
        srt = np.sort(logits[0])[::-1]
        assert srt[s.top_k - 1] > srt[s.top_k], f"layer {l}: exact tie at the top-k boundary"
        xs_o.append(xn)
        idx_o.append(idx)

    # teacher forcing: layer l of the GPU path from the oracle's x_l
    worst = 0.0
    for l in range(L):
        x = torch.from_numpy(xs_o[l]).cuda()
        idx = gpu_layer(l, x)
        assert np.array_equal(idx, idx_o[l]), f"layer {l}: selected experts differ"
        y_gpu = x.cpu().numpy() - xs_o[l]
        y_ref = xs_o[l + 1] - xs_o[l]
        rel, mx = y_errors(y_gpu, y_ref)
        print(f"layer {l:2d}: rel L2 {rel:.2e}  max/rms {mx:.2e}")
        worst = max(worst, rel)
        assert_y_close(y_gpu, y_ref)

    # free running: same experts at every layer
    x = torch.from_numpy(x0).cuda()
    for l in range(L):
        idx = gpu_layer(l, x)
        assert np.array_equal(idx, idx_o[l]), f"free-running layer {l}: selected experts differ"
    st, bits = B.coli_moe_read_status(bufs.ws)
    assert st == B.COLI_OK and bits == 0
    rel, mx = y_errors(x.cpu().numpy(), xs_o[-1])
    print(f"free-running final x: rel L2 {rel:.2e}  max/rms {mx:.2e}  (worst layer {worst:.2e})")
    # the oracle's own chain amplifies a 2^-24 input change only to ~4e-7 over 16 layers,
    # so the free-running stack is held to the per-layer bar as well
    assert_y_close(x.cpu().numpy(), xs_o[-1])

    # the same 16 layers as one resident launch (coli_moe_stack)
    ws = torch.zeros(B.coli_moe_workspace_bytes(dims, T), dtype=torch.uint8, device="cuda")
    B.check(B.coli_moe_workspace_init(ws))
    y = torch.empty(T, s.hidden, device="cuda")
    idx_all = torch.full((L, T, s.top_k), -1, dtype=torch.int32, device="cuda")
    B.check(B.coli_moe_stack(dims, [lay[4] for lay in layers], [gamma] * L, 1e-5,
                             torch.from_numpy(x0).cuda(), T, idx_all, y, ws), "coli_moe_stack")
    for l in range(L):
        assert np.array_equal(idx_all[l].cpu().numpy(), idx_o[l]), f"stack launch layer {l}: experts differ"
    rel, mx = y_errors(y.cpu().numpy(), xs_o[-1])
    print(f"one-launch stack final x: rel L2 {rel:.2e}  max/rms {mx:.2e}")
    assert_y_close(y.cpu().numpy(), xs_o[-1])
    st, bits = B.coli_moe_read_status(ws)
    assert st == B.COLI_OK and bits == 0
