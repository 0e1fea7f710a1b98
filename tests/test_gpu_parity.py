"""Parity of the CUDA library (through the C ABI) against the CPU oracle.

Indices, unions and assignment lists must match bit for bit; logits must be equal
floats; routing weights within 1e-6; y within relative L2 1e-4 and max |diff| within
1e-3 * rms(y_oracle) (fp32 contract).
"""
import numpy as np
import pytest
import torch

import oracle
from int4_routed_expert_gemv_b200 import binding as B
from int4_routed_expert_gemv_b200 import synth
from layers import (W_ABS, assert_route_union_equal, assert_y_close, host_outputs,
                    make_device_layer, oracle_layer, run_layer)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib(colimoe):
    assert torch.cuda.is_available()
    return colimoe


def _x(shape, seed, T, variant):
    return synth.activations(shape, seed, T, variant)


def test_generator_same_bytes_on_device_and_host():
    for shape in [synth.SMALL, synth.GLM]:
        for e in [0, shape.n_experts]:
            a = synth.expert_blob(shape, 1, 2, e, device="cuda").cpu()
            b = synth.expert_blob(shape, 1, 2, e, device="cpu")
            assert torch.equal(a, b)


@pytest.mark.parametrize("name", ["moe_h1024_i512_e64_k4_t1", "moe_h1024_i512_e64_k4_t4_zipf"])
def test_small_layer_full_parity(name):
    wl = synth.WORKLOADS[name]
    L = make_device_layer(wl.shape, wl.seed, zipf=wl.zipf)
    x = _x(wl.shape, wl.seed, wl.tokens, wl.x_variant)
    got = run_layer(L, torch.from_numpy(x).cuda(), wl.tokens)
    ref = oracle_layer(L, x)
    assert_route_union_equal(got, ref)
    assert_y_close(got["y"], ref["y"])


@pytest.mark.parametrize("name", ["glm52_moe_h6144_i2048_e256_k8_t1",
                                  "glm52_moe_h6144_i2048_e256_k8_t4_zipf"])
def test_glm_layer_full_parity(name):
    wl = synth.WORKLOADS[name]
    L = make_device_layer(wl.shape, wl.seed, zipf=wl.zipf)
    x = _x(wl.shape, wl.seed, wl.tokens, wl.x_variant)
    got = run_layer(L, torch.from_numpy(x).cuda(), wl.tokens)
    ref = oracle_layer(L, x)
    assert_route_union_equal(got, ref)
    assert_y_close(got["y"], ref["y"])


@pytest.mark.parametrize("T", [2, 3, 5, 8, 9, 37])
def test_ragged_batches(T):
    shape = synth.SMALL
    L = make_device_layer(shape, 11, zipf=True)
    x = _x(shape, 11, T, 7)
    got = run_layer(L, torch.from_numpy(x).cuda(), T)
    ref = oracle_layer(L, x)
    assert_route_union_equal(got, ref)
    assert_y_close(got["y"], ref["y"])


@pytest.mark.parametrize("H,I,E,k,ns", [(64, 64, 4, 1, 1), (64, 64, 4, 4, 1), (128, 256, 8, 3, 0),
                                        (256, 128, 16, 2, 1), (512, 64, 6, 6, 0),
                                        (2048, 1024, 32, 8, 1), (64, 64, 1024, 32, 1),
                                        (128, 64, 1024, 32, 1), (3072, 192, 96, 5, 1),
                                        (4096, 128, 8, 2, 0)])
@pytest.mark.parametrize("T", [1, 3, 4])
def test_shapes_and_edges(H, I, E, k, ns, T):
    shape = synth.LayerShape(H, I, E, k, ns)
    L = make_device_layer(shape, 21 + H + I + E, zipf=(E % 2 == 0))
    x = _x(shape, 5, T, 3)
    got = run_layer(L, torch.from_numpy(x).cuda(), T)
    ref = oracle_layer(L, x)
    assert_route_union_equal(got, ref)
    assert_y_close(got["y"], ref["y"])


def test_ties_go_to_lower_index():
    shape = synth.LayerShape(256, 128, 16, 4, 1)
    wr = np.zeros((16, 256), np.float32)                 # all logits equal
    L = make_device_layer(shape, 3, w_router_host=wr)
    x = _x(shape, 3, 2, 0)
    got = run_layer(L, torch.from_numpy(x).cuda(), 2)
    assert got["idx"].tolist() == [[0, 1, 2, 3]] * 2
    assert np.all(got["w"] == np.float32(0.25))
    ref = oracle_layer(L, x)
    assert_route_union_equal(got, ref)
    assert_y_close(got["y"], ref["y"])
    # duplicated router rows: equal logits, the lower index first
    wr = synth.router_weight(shape, 9)
    wr[7] = wr[2]
    wr[12] = wr[2]
    L = make_device_layer(shape, 3, w_router_host=wr * 8)
    x = np.tile(wr[2:3] * 50, (1, 1)).astype(np.float32)
    got = run_layer(L, torch.from_numpy(x).cuda(), 1)
    ref = oracle_layer(L, x)
    assert got["idx"][0, :3].tolist() == [2, 7, 12]
    assert_route_union_equal(got, ref)


def test_separate_calls_and_residual():
    wl = synth.WORKLOADS["moe_h1024_i512_e64_k4_t4_zipf"]
    L = make_device_layer(wl.shape, wl.seed, zipf=True)
    T = 4
    x = _x(wl.shape, wl.seed, T, 5)
    ref = oracle_layer(L, x)
    bufs = B.LayerBuffers(L.dims, T)
    xd = torch.from_numpy(x).cuda()
    B.check(B.coli_moe_route(L.dims, L.w_router, L.bias, xd, T, bufs.idx, bufs.w, bufs.logits,
                             bufs.ws))
    # union from the oracle's selection (an input, not an output of the device path)
    idx_in = torch.from_numpy(ref["idx"]).cuda()
    B.check(B.coli_moe_union(L.dims, idx_in, T, bufs.union_ids, bufs.n_union, bufs.offsets,
                             bufs.assign, bufs.ws))
    got = host_outputs(bufs, T, wl.shape)
    assert_route_union_equal(got, ref)
    # forward from the oracle's routing, with a residual
    res = synth.activations(wl.shape, 77, T, 0)
    resd = torch.from_numpy(res).cuda()
    w_in = torch.from_numpy(ref["w"]).cuda()
    B.check(B.coli_moe_forward(L.dims, L.weights, xd, T, idx_in, w_in, bufs.union_ids,
                               bufs.n_union, bufs.offsets, bufs.assign, resd, bufs.y, bufs.ws))
    y = bufs.y[:T].cpu().numpy()
    assert_y_close(y - res, ref["y"])
    # gate_up + down halves, residual aliasing y
    bufs.y[:T].copy_(resd)
    B.check(B.coli_moe_gate_up(L.dims, L.weights, xd, T, bufs.union_ids, bufs.n_union,
                               bufs.offsets, bufs.assign, bufs.ws))
    B.check(B.coli_moe_down(L.dims, L.weights, T, w_in, bufs.union_ids, bufs.n_union,
                            bufs.offsets, bufs.assign, bufs.y, bufs.y, bufs.ws))
    assert_y_close(bufs.y[:T].cpu().numpy() - res, ref["y"])
    st, bits = B.coli_moe_read_status(bufs.ws)
    assert st == B.COLI_OK and bits == 0


def test_zero_tokens_is_a_noop():
    shape = synth.SMALL
    L = make_device_layer(shape, 0)
    bufs = B.LayerBuffers(L.dims, 1)
    bufs.y.fill_(7.0)
    x = torch.zeros(1, shape.hidden, device="cuda")
    B.check(B.coli_moe_layer(L.dims, L.weights, x, 0, bufs.idx, bufs.w, bufs.logits,
                             bufs.union_ids, bufs.n_union, bufs.offsets, bufs.assign, None,
                             bufs.y, bufs.ws))
    torch.cuda.synchronize()
    assert torch.all(bufs.y == 7.0)


def test_device_errors_are_flagged_not_faulted():
    shape = synth.LayerShape(256, 128, 16, 4, 1)
    L = make_device_layer(shape, 4)
    bufs = B.LayerBuffers(L.dims, 2)
    x = torch.from_numpy(_x(shape, 4, 2, 0)).cuda()
    x[1, 17] = float("nan")
    B.check(B.coli_moe_route(L.dims, L.w_router, None, x, 2, bufs.idx, bufs.w, bufs.logits,
                             bufs.ws))
    st, bits = B.coli_moe_read_status(bufs.ws)
    assert st == B.COLI_EDEVICE and bits & B.DEV_NONFINITE
    B.check(B.coli_moe_workspace_init(bufs.ws))
    assert B.coli_moe_read_status(bufs.ws) == (B.COLI_OK, 0)
    bad = torch.tensor([[0, 3, 3, 1], [2, 99, 1, 0]], dtype=torch.int32, device="cuda")
    B.check(B.coli_moe_union(L.dims, bad, 2, bufs.union_ids, bufs.n_union, bufs.offsets,
                             bufs.assign, bufs.ws))
    st, bits = B.coli_moe_read_status(bufs.ws)
    assert st == B.COLI_EDEVICE and bits & B.DEV_BAD_INDEX


def test_rmsnorm_matches_oracle():
    H, T = 6144, 3
    x = synth.activations(synth.GLM, 2, T, 4) * 3
    g = np.ones(H, np.float32)
    out = torch.empty(T, H, device="cuda")
    B.check(B.coli_rmsnorm(H, T, torch.from_numpy(x).cuda(), torch.from_numpy(g).cuda(), 1e-5, out))
    ref = oracle.rmsnorm(x, g, 1e-5)
    got = out.cpu().numpy()
    assert np.max(np.abs(got.view(np.int32) - ref.view(np.int32))) <= 1


@pytest.mark.parametrize("scale", [4.0, 16.0])
def test_large_activations_tiny_negative_h(scale):
    # large x drives many gate values far negative: silu(g) * u is then a tiny negative
    # number, the case where a floor-digit split of h can round up to the next integer
    shape = synth.LayerShape(1024, 512, 64, 4, 1)
    L = make_device_layer(shape, 13)
    x = (synth.activations(shape, 13, 3, 2) * scale).astype(np.float32)
    got = run_layer(L, torch.from_numpy(x).cuda(), 3)
    ref = oracle_layer(L, x)
    assert_route_union_equal(got, ref)
    assert_y_close(got["y"], ref["y"], rel_l2=1e-5)


@pytest.mark.parametrize("H,I,E,k,T", [(1024, 512, 64, 4, 1), (1024, 512, 64, 4, 4),
                                       (1024, 512, 64, 4, 8), (1024, 512, 64, 4, 9),
                                       (4096, 256, 16, 4, 7), (4096, 256, 16, 4, 8),
                                       (4096, 256, 16, 4, 12)])
def test_layer_call_equals_separate_calls(H, I, E, k, T):
    # Decode batches (T <= 4) run coli_moe_layer as one fused launch (tensor-core int8
    # tiles); larger batches form the activation digits in a launch of their own (T <= 8)
    # or stage x before the router has finished, while the separate calls form them inside
    # gate/up.  Routing, union and assignment lists must agree bit for bit either way; y is
    # bit-equal where both take the same kernels and within the oracle bar otherwise.
    shape = synth.LayerShape(H, I, E, k, 1)
    L = make_device_layer(shape, 40 + T, zipf=True)
    x = _x(shape, 40 + T, T, 6)
    xd = torch.from_numpy(x).cuda()
    got = run_layer(L, xd, T)
    ref = oracle_layer(L, x)
    assert_route_union_equal(got, ref)
    assert_y_close(got["y"], ref["y"])
    bufs = B.LayerBuffers(L.dims, T)
    B.check(B.coli_moe_route_union(L.dims, L.w_router, L.bias, xd, T, bufs.idx, bufs.w,
                                   bufs.logits, bufs.union_ids, bufs.n_union, bufs.offsets,
                                   bufs.assign, bufs.ws))
    B.check(B.coli_moe_gate_up(L.dims, L.weights, xd, T, bufs.union_ids, bufs.n_union,
                               bufs.offsets, bufs.assign, bufs.ws))
    B.check(B.coli_moe_down(L.dims, L.weights, T, bufs.w, bufs.union_ids, bufs.n_union,
                            bufs.offsets, bufs.assign, None, bufs.y, bufs.ws))
    sep = host_outputs(bufs, T, shape)
    keys = ("idx", "logits", "union_ids", "offsets", "assign") + (("w", "y") if T > 4 else ())
    for key in keys:
        assert np.array_equal(got[key], sep[key]), key
    assert np.abs(got["w"] - sep["w"]).max() <= W_ABS
    assert_y_close(sep["y"], ref["y"])
    assert got["n_union"] == sep["n_union"]
    st, bits = B.coli_moe_read_status(bufs.ws)
    assert st == B.COLI_OK and bits == 0
