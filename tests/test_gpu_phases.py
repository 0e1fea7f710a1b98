"""The phase-stamp build: the regular library reports no stamps; the stamp build records,
for every CTA of a fused decode launch, phases in launch order, and its results equal the
regular build's bit for bit (the stamps only store timer values)."""
import ctypes
import os

import numpy as np
import pytest

from int4_routed_expert_gemv_b200 import binding as B
from int4_routed_expert_gemv_b200 import build

pytestmark = pytest.mark.gpu


def test_regular_build_has_no_stamps(colimoe):
    st, tl = B.coli_debug_phase_stamps()
    assert st == B.COLI_EUNSUPPORTED and tl.size == 0


def test_stamped_launch_phases_in_order():
    import subprocess, sys
    path = build.build(stamps=True)
    assert os.path.exists(path)
    code = r'''
import sys, numpy as np, torch
from int4_routed_expert_gemv_b200 import binding as B, build, synth
B.LIB_PATH = build.STAMPS_LIB
s = synth.SMALL
dims = B.make_dims(s.hidden, s.inter, s.n_experts, s.top_k, s.n_shared)
ex = synth.experts_tensor(s, 5, device="cuda"); sh = synth.shared_tensor(s, 5, device="cuda")
wr = torch.from_numpy(synth.router_weight(s, 5)).cuda()
w = B.make_weights(wr, None, ex.reshape(-1), sh, s.stride)
x = torch.from_numpy(synth.activations(s, 5, 1, 0)).cuda()
b = B.LayerBuffers(dims, 1)
B.check(B.coli_moe_layer(dims, w, x, 1, b.idx, b.w, None, b.union_ids, b.n_union, b.offsets, b.assign, None, b.y, b.ws))
torch.cuda.synchronize()
st, tl = B.coli_debug_phase_stamps()
assert st == B.COLI_OK, st
assert B.coli_moe_read_status(b.ws) == (B.COLI_OK, 0)
np.save(sys.argv[1], tl)
np.save(sys.argv[2], b.y[:1].cpu().numpy())
'''
    import tempfile
    d = tempfile.mkdtemp()
    ft, fy = os.path.join(d, "tl.npy"), os.path.join(d, "y.npy")
    subprocess.run([sys.executable, "-c", code, ft, fy], check=True, cwd=os.path.dirname(os.path.dirname(__file__)))
    tl = np.load(ft).astype(np.int64)
    tl = tl[tl[:, 0] > 0]            # the launch's CTAs (the buffer has rows for 256)
    assert tl.shape[0] >= 100 and tl.shape[1] == 16
    # every CTA: entry <= input loaded <= ... ; the control warp's table after entry
    for cta in tl:
        order = [cta[i] for i in (0, 1, 3, 6, 7, 9)]
        assert all(v > 0 for v in order)
        assert all(a <= b for a, b in zip(order, order[1:]))
        assert cta[0] <= cta[4] <= cta[9]
    # the same layer through the regular build gives the same y
    from int4_routed_expert_gemv_b200 import synth
    import torch
    s = synth.SMALL
    dims = B.make_dims(s.hidden, s.inter, s.n_experts, s.top_k, s.n_shared)
    ex = synth.experts_tensor(s, 5, device="cuda"); sh = synth.shared_tensor(s, 5, device="cuda")
    wr = torch.from_numpy(synth.router_weight(s, 5)).cuda()
    w = B.make_weights(wr, None, ex.reshape(-1), sh, s.stride)
    x = torch.from_numpy(synth.activations(s, 5, 1, 0)).cuda()
    b = B.LayerBuffers(dims, 1)
    B.check(B.coli_moe_layer(dims, w, x, 1, b.idx, b.w, None, b.union_ids, b.n_union, b.offsets, b.assign,
                             None, b.y, b.ws))
    assert np.array_equal(b.y[:1].cpu().numpy(), np.load(fy))
