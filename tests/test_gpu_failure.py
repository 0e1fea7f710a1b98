"""The failure path of the library's bounded device waits, on the GPU, without a fault.

coli_debug_wait_timeout runs one wait of the kind every kernel of the library uses (an
mbarrier, polled with a cycle budget) on a barrier nothing ever arrives at, with a budget
of a few thousand cycles.  Checked: the kernel returns, the workspace status word reports
COLI_DEV_TIMEOUT with the wait's site, coli_moe_read_status maps it to COLI_ETIMEOUT, and
the stream and context are usable afterwards (workspace init clears the status and a
routing call runs and matches the oracle).
"""
import numpy as np
import pytest
import torch

import oracle
from int4_routed_expert_gemv_b200 import binding as B
from int4_routed_expert_gemv_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("budget", [2000, 200000])
def test_bounded_wait_runs_out_and_reports(colimoe, budget):
    shape = synth.LayerShape(hidden=128, inter=64, n_experts=8, top_k=2, n_shared=1)
    dims = B.make_dims(shape.hidden, shape.inter, shape.n_experts, shape.top_k, shape.n_shared)
    ws = torch.zeros(B.coli_moe_workspace_bytes(dims, 4), dtype=torch.uint8, device="cuda")
    B.check(B.coli_moe_workspace_init(ws))
    returned = torch.zeros(1, dtype=torch.int32, device="cuda")
    B.check(B.coli_debug_wait_timeout(ws, budget, returned), "coli_debug_wait_timeout")
    torch.cuda.synchronize()
    assert int(returned.item()) == 1          # the wait gave up and the kernel ended
    st, bits = B.coli_moe_read_status(ws)
    assert st == B.COLI_ETIMEOUT and bits & B.DEV_TIMEOUT
    site = int(ws[12:16].cpu().view(torch.int32).item())   # header word 3: timeout site
    assert site == 99

    # the context is still usable: clear the status and run a routing call
    B.check(B.coli_moe_workspace_init(ws))
    assert B.coli_moe_read_status(ws) == (B.COLI_OK, 0)
    T = 3
    wr_h = synth.router_weight(shape, 5)
    x_h = synth.activations(shape, 5, T)
    idx = torch.empty(T, shape.top_k, dtype=torch.int32, device="cuda")
    w = torch.empty(T, shape.top_k, device="cuda")
    B.check(B.coli_moe_route(dims, torch.from_numpy(wr_h).cuda(), None, torch.from_numpy(x_h).cuda(), T,
                             idx, w, None, ws))
    idx_o, w_o, _ = oracle.route(x_h, wr_h, None, shape.top_k)
    assert np.array_equal(idx.cpu().numpy(), idx_o)
    assert B.coli_moe_read_status(ws) == (B.COLI_OK, 0)


def test_bad_arguments_rejected_on_the_host(colimoe):
    ws = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    returned = torch.zeros(1, dtype=torch.int32, device="cuda")
    assert B.coli_debug_wait_timeout(ws, 0, returned) == B.COLI_EINVAL
    assert B.coli_debug_wait_timeout(ws, (1 << 32) + 1, returned) == B.COLI_EINVAL
