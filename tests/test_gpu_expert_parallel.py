"""Expert parallelism through the library on one GPU: the ranks of a W-way split are run one
after another (no collective), each with only its experts' blobs, and their shares of y,
added on the host in rank order (what the all-reduce does), match the oracle.  The
restriction kernel's lists equal the reference restriction of test_expert_parallel bit for
bit, and a rank whose range holds none of the batch's experts contributes exactly zero.
"""
import numpy as np
import pytest
import torch

import oracle
from int4_routed_expert_gemv_b200 import binding as B
from int4_routed_expert_gemv_b200 import synth
from int4_routed_expert_gemv_b200.expert_parallel import LibraryBackend, expert_range
from layers import assert_y_close
from test_expert_parallel import restrict

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name,world", [("moe_h1024_i512_e64_k4_t4_zipf", 2),
                                        ("moe_h1024_i512_e64_k4_t4_zipf", 4),
                                        ("moe_h1024_i512_e64_k4_t1", 3),
                                        ("glm52_moe_h6144_i2048_e256_k8_t1", 2)])
def test_ranks_add_up_to_the_layer(colimoe, name, world):
    wl = synth.WORKLOADS[name]
    s, T = wl.shape, wl.tokens
    if s.hidden > 1024:
        s = synth.LayerShape(s.hidden, s.inter, 32, s.top_k, s.n_shared)   # 32 of the GLM experts
    experts = synth.experts_tensor(s, wl.seed, device="cuda")
    shared = synth.shared_tensor(s, wl.seed, device="cuda")
    wr_h = synth.router_weight(s, wl.seed)
    bias_h = synth.zipf_bias(s.n_experts) if wl.zipf else None
    wr = torch.from_numpy(wr_h).cuda()
    bias = torch.from_numpy(bias_h).cuda() if wl.zipf else None
    x_h = synth.activations(s, wl.seed, T, 17)
    x = torch.from_numpy(x_h).cuda()
    y_sum = np.zeros((T, s.hidden), np.float32)
    for r in range(world):
        e0, e1 = expert_range(s.n_experts, world, r)
        be = LibraryBackend(s.hidden, s.inter, s.n_experts, s.top_k, e0, e1, r == 0, T, "cuda")
        local = B.make_weights(wr, bias, experts[e0:e1].reshape(-1), shared if r == 0 else None, s.stride)
        rt = be.route(wr, bias, x, T)
        rl = be.restrict(rt, T, e0, e1)
        y = torch.full((T, s.hidden), float("nan"), device="cuda")
        be.forward(local, x, T, rl, None, y)
        assert B.coli_moe_read_status(be.ws_l) == (B.COLI_OK, 0)
        ref = restrict(rt.union_ids.cpu().numpy(), rt.n_union.cpu().numpy()[0], rt.offsets.cpu().numpy(),
                       rt.assign.cpu().numpy(), e0, e1, s.n_experts, T * s.top_k)
        got = (rl.union_ids.cpu().numpy(), rl.n_union.cpu().numpy()[0], rl.offsets.cpu().numpy(),
               rl.assign.cpu().numpy())
        nl = int(ref[1])
        assert got[1] == ref[1]
        assert np.array_equal(got[0], ref[0]) and np.array_equal(got[2], ref[2])
        assert np.array_equal(got[3][:ref[2][nl]], ref[3][:ref[2][nl]])
        yh = y.cpu().numpy()
        if nl == 0 and r != 0:
            assert np.array_equal(yh, np.zeros_like(yh))
        y_sum += yh
    idx, w, _ = oracle.route(x_h, wr_h, bias_h, s.top_k)
    blobs = {int(e): experts[int(e), :s.blob_bytes].cpu().numpy() for e in np.unique(idx)}
    y_ref = oracle.forward_sparse(s.hidden, s.inter, s.top_k, 1, x_h, blobs,
                                  shared[:s.blob_bytes].cpu().numpy(), idx, w)
    assert_y_close(y_sum, y_ref)


def test_restrict_rejects_bad_ranges(colimoe):
    dims = B.make_dims(1024, 512, 16, 2, 1)
    i = torch.zeros(64, dtype=torch.int32, device="cuda")
    assert B.coli_moe_union_restrict(dims, 4, 4, 4, i, i, i, i, i, i, i, i) == B.COLI_EINVAL
    assert B.coli_moe_union_restrict(dims, 4, 0, 17, i, i, i, i, i, i, i, i) == B.COLI_EINVAL
    assert B.coli_moe_union_restrict(dims, 4, -1, 3, i, i, i, i, i, i, i, i) == B.COLI_EINVAL
