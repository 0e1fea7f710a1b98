"""coli_moe_forward_fmt (gs64 int8, per-row int4, gs64 int2, and gs64 int4 through the same
kernels) against the oracle's orc_forward_fmt, through the C ABI.

Weights: random payload bytes (every code of the container equally likely) and fp16 scales
~U[0.005, 0.02], generated on the host.  Routing by the library's router on the seeded
layer; y within relative L2 1e-4 and max 1e-3 rms of the oracle; idx bit-exact.
"""
import numpy as np
import pytest
import torch

import oracle
from int4_routed_expert_gemv_b200 import binding as B
from int4_routed_expert_gemv_b200 import synth
from layers import assert_y_close

pytestmark = pytest.mark.gpu

FMTS = [B.FMT_INT4_G64, B.FMT_INT8_G64, B.FMT_INT4_ROW, B.FMT_INT2_G64]
BITS = {B.FMT_INT4_G64: 4, B.FMT_INT8_G64: 8, B.FMT_INT4_ROW: 4, B.FMT_INT2_G64: 2}


def random_blob(rng, H, I, fmt):
    b = BITS[fmt]
    payload = rng.integers(0, 256, 3 * H * I * b // 8, dtype=np.uint8)
    if fmt == B.FMT_INT4_ROW:
        n_sc = 2 * I + H
    else:
        n_sc = 2 * I * (H // 64) + H * (I // 64)
    sc = rng.uniform(0.005, 0.02, n_sc).astype(np.float16).view(np.uint8)
    blob = np.concatenate([payload, sc])
    assert blob.size == B.coli_moe_blob_bytes_fmt(H, I, fmt) == oracle.blob_bytes_fmt(H, I, fmt)
    return blob


def run_fmt(shape, fmt, T, seed, zipf, residual):
    H, I, E, k = shape.hidden, shape.inter, shape.n_experts, shape.top_k
    rng = np.random.default_rng(seed * 10 + fmt)
    blob_bytes = B.coli_moe_blob_bytes_fmt(H, I, fmt)
    stride = (blob_bytes + 255) // 256 * 256
    host = np.zeros((E, stride), np.uint8)
    for e in range(E):
        host[e, :blob_bytes] = random_blob(rng, H, I, fmt)
    shared_h = np.zeros(stride, np.uint8)
    shared_h[:blob_bytes] = random_blob(rng, H, I, fmt)
    experts = torch.from_numpy(host).cuda()
    shared = torch.from_numpy(shared_h).cuda()
    wr_h = synth.router_weight(shape, seed)
    bias_h = synth.zipf_bias(E) if zipf else None
    wr = torch.from_numpy(wr_h).cuda()
    bias = torch.from_numpy(bias_h).cuda() if zipf else None
    dims = B.make_dims(H, I, E, k, shape.n_shared)
    weights = B.make_weights(wr, bias, experts, shared, stride)
    x_h = synth.activations(shape, seed, T, 77 + fmt)
    res_h = synth.activations(shape, seed + 1, T, 5) if residual else None
    x = torch.from_numpy(x_h).cuda()
    bufs = B.LayerBuffers(dims, T)
    B.check(B.coli_moe_route_union(dims, wr, bias, x, T, bufs.idx, bufs.w, None, bufs.union_ids, bufs.n_union,
                                   bufs.offsets, bufs.assign, bufs.ws))
    y = torch.full((T, H), float("nan"), device="cuda")
    B.check(B.coli_moe_forward_fmt(dims, fmt, weights, x, T, bufs.w, bufs.union_ids, bufs.n_union, bufs.offsets,
                                   bufs.assign, None if res_h is None else torch.from_numpy(res_h).cuda(), y,
                                   bufs.ws), "coli_moe_forward_fmt")
    assert B.coli_moe_read_status(bufs.ws) == (B.COLI_OK, 0)
    idx, w, _ = oracle.route(x_h, wr_h, bias_h, k)
    assert np.array_equal(bufs.idx[:T].cpu().numpy(), idx)
    blobs = {int(e): host[int(e), :blob_bytes] for e in np.unique(idx)}
    y_ref = oracle.forward_sparse_fmt(H, I, k, shape.n_shared, fmt, x_h, blobs, shared_h[:blob_bytes], idx, w)
    if res_h is not None:
        y_ref = y_ref + res_h
    return y.cpu().numpy(), y_ref


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("T,zipf,residual", [(1, False, False), (4, True, True), (3, True, False)])
def test_formats_small_layer(colimoe, fmt, T, zipf, residual):
    shape = synth.LayerShape(1024, 512, 64, 4, 1)
    y, y_ref = run_fmt(shape, fmt, T, 3, zipf, residual)
    rel, mx = assert_y_close(y, y_ref)
    print(f"fmt {fmt} T={T}: rel L2 {rel:.2e} max/rms {mx:.2e}")


@pytest.mark.parametrize("fmt", FMTS)
def test_formats_wide_and_ragged_shapes(colimoe, fmt):
    # hidden not a multiple of 1024, intermediate 192: ragged chunk counts per lane
    shape = synth.LayerShape(3072, 192, 24, 5, 1)
    y, y_ref = run_fmt(shape, fmt, 2, 8, True, False)
    assert_y_close(y, y_ref)


def test_formats_glm_shape_int8(colimoe):
    y, y_ref = run_fmt(synth.LayerShape(6144, 2048, 32, 8, 1), B.FMT_INT8_G64, 1, 1, False, False)
    assert_y_close(y, y_ref)


def test_formats_bad_arguments(colimoe):
    shape = synth.LayerShape(1024, 512, 8, 2, 1)
    dims = B.make_dims(1024, 512, 8, 2, 1)
    bufs = B.LayerBuffers(dims, 5)
    d = torch.zeros(4096, device="cuda")
    blob = B.coli_moe_blob_bytes_fmt(1024, 512, B.FMT_INT8_G64)
    ex = torch.zeros(8 * ((blob + 255) // 256 * 256), dtype=torch.uint8, device="cuda")
    w = B.make_weights(d, None, ex, ex, (blob + 255) // 256 * 256)
    args = (d, 1, bufs.w, bufs.union_ids, bufs.n_union, bufs.offsets, bufs.assign, None, d, bufs.ws)
    assert B.coli_moe_forward_fmt(dims, 7, w, *args) == B.COLI_EINVAL
    assert B.coli_moe_forward_fmt(dims, B.FMT_INT8_G64, w, d, 5, *args[2:]) == B.COLI_EUNSUPPORTED
    small = B.make_weights(d, None, ex, ex, 256)     # stride below the blob size
    assert B.coli_moe_forward_fmt(dims, B.FMT_INT8_G64, small, *args) == B.COLI_EINVAL
    assert B.coli_moe_blob_bytes_fmt(1024, 512, 9) == 0
