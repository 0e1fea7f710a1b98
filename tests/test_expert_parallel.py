"""Expert parallelism on the CPU: two gloo ranks run ExpertParallelLayer (the module's
partition, union restriction and all-reduce of y) with an oracle-backed compute backend,
and the combined y equals the whole layer's oracle y within float rounding.

The backend follows the library's contract step by step: routing and union over all E
experts (oracle.route, oracle.union), the restriction to the rank's range (the reference
`restrict` below, which also pins the semantics the CUDA kernel is checked against on the
GPU), and the rank's share of y from the restricted lists (oracle experts).
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle
from int4_routed_expert_gemv_b200 import synth
from int4_routed_expert_gemv_b200.expert_parallel import ExpertParallelLayer, Routing, expert_range

SHAPE = synth.LayerShape(hidden=128, inter=64, n_experts=12, top_k=3, n_shared=1)
SEED = 21


def restrict(union_ids, n_union, offsets, assign, e0, e1, E, Tk):
    """Union entries of experts [e0, e1), renumbered; the library's coli_moe_union_restrict."""
    nu = int(n_union)
    keep = [u for u in range(nu) if e0 <= union_ids[u] < e1]
    El = e1 - e0
    uid = np.full(El, -1, np.int32)
    off = np.zeros(El + 1, np.int32)
    asg = np.zeros(Tk, np.int32)
    pos = 0
    for j, u in enumerate(keep):
        uid[j] = union_ids[u] - e0
        off[j] = pos
        seg = assign[offsets[u]:offsets[u + 1]]
        asg[pos:pos + len(seg)] = seg
        pos += len(seg)
    off[len(keep):] = pos
    return uid, np.int32(len(keep)), off, asg


class OracleBackend:
    def __init__(self, blobs, shared, e0):
        self.blobs, self.shared, self.e0 = blobs, shared, e0

    def route(self, w_router, bias, x, T):
        s = SHAPE
        idx, w, _ = oracle.route(x.numpy(), w_router, bias, s.top_k)
        uid, nu, off, asg = oracle.union(idx, s.n_experts)
        t = lambda a: torch.from_numpy(np.asarray(a))
        return Routing(t(idx), t(w), t(uid), t(np.array([nu], np.int32)), t(off), t(asg))

    def restrict(self, r, T, e0, e1):
        s = SHAPE
        uid, nu, off, asg = restrict(r.union_ids.numpy(), r.n_union.numpy()[0], r.offsets.numpy(), r.assign.numpy(),
                                     e0, e1, s.n_experts, T * s.top_k)
        t = lambda a: torch.from_numpy(np.asarray(a))
        return Routing(r.idx, r.w, t(uid), t(np.array([nu], np.int32)), t(off), t(asg))

    def forward(self, weights, x, T, r, residual, y):
        s = SHAPE
        xh = x.numpy()
        acc = np.zeros((T, s.hidden))
        if self.shared is not None:
            for t in range(T):
                out, _ = oracle.expert(s.hidden, s.inter, self.shared, xh[t])
                acc[t] += out
        w = r.w.numpy().reshape(-1)
        nu = int(r.n_union.numpy()[0])
        for u in range(nu):
            e = self.e0 + int(r.union_ids[u])
            for a in r.assign.numpy()[r.offsets[u]:r.offsets[u + 1]]:
                out, _ = oracle.expert(s.hidden, s.inter, self.blobs[e], xh[a // s.top_k])
                acc[a // s.top_k] += float(w[a]) * out
        if residual is not None:
            acc += residual.numpy()
        y.copy_(torch.from_numpy(acc.astype(np.float32)))


def layer_inputs():
    s = SHAPE
    experts = synth.experts_tensor(s, SEED).numpy()
    blobs = {e: experts[e, :s.blob_bytes] for e in range(s.n_experts)}
    shared = synth.shared_tensor(s, SEED).numpy()[:s.blob_bytes]
    wr = synth.router_weight(s, SEED) * 4.0
    bias = synth.zipf_bias(s.n_experts)
    x = synth.activations(s, SEED, 3, 1)
    res = synth.activations(s, SEED + 1, 3, 2)
    return experts, blobs, shared, wr, bias, x, res


def _rank(rank, world, port, q):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        experts, blobs, shared, wr, bias, x, res = layer_inputs()
        e0, e1 = expert_range(SHAPE.n_experts, world, rank)
        be = OracleBackend(blobs, shared if rank == 0 else None, e0)
        L = ExpertParallelLayer(SHAPE.n_experts, wr, bias, None, be)
        y = L.forward(torch.from_numpy(x), 3, torch.from_numpy(res))
        q.put((rank, y.numpy()))
    finally:
        dist.destroy_process_group()


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("world", [2, 3])
def test_expert_parallel_ranks_add_up_to_the_layer(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = free_port()
    ps = [ctx.Process(target=_rank, args=(r, world, port, q)) for r in range(world)]
    for p in ps:
        p.start()
    outs = dict(q.get(timeout=120) for _ in range(world))
    for p in ps:
        p.join(timeout=60)
        assert p.exitcode == 0
    experts, blobs, shared, wr, bias, x, res = layer_inputs()
    s = SHAPE
    idx, w, _ = oracle.route(x, wr, bias, s.top_k)
    y_ref = oracle.forward(s.hidden, s.inter, s.n_experts, s.top_k, 1, x, experts, s.stride, shared, idx, w) + res
    for r in range(world):
        assert np.array_equal(outs[r], outs[0])          # every rank holds the sum
        rel = np.linalg.norm(outs[r] - y_ref) / np.linalg.norm(y_ref)
        assert rel < 1e-6, rel


def test_expert_range_covers_every_expert_once():
    for E in (8, 12, 256):
        for W in (1, 2, 3, 8):
            ranges = [expert_range(E, W, r) for r in range(W)]
            assert ranges[0][0] == 0 and ranges[-1][1] == E
            assert all(a[1] == b[0] for a, b in zip(ranges, ranges[1:]))
            assert max(b - a for a, b in ranges) - min(b - a for a, b in ranges) <= 1
    with pytest.raises(ValueError):
        expert_range(2, 3, 0)


def test_restrict_reference_partitions_the_union():
    """Over all ranks the restricted lists hold every (token, slot) exactly once."""
    s = SHAPE
    rng = np.random.default_rng(3)
    T = 5
    idx = np.stack([rng.choice(s.n_experts, s.top_k, replace=False) for _ in range(T)]).astype(np.int32)
    uid, nu, off, asg = oracle.union(idx, s.n_experts)
    seen = []
    for r in range(3):
        e0, e1 = expert_range(s.n_experts, 3, r)
        ul, nl, ol, al = restrict(uid, nu, off, asg, e0, e1, s.n_experts, T * s.top_k)
        for j in range(nl):
            for a in al[ol[j]:ol[j + 1]]:
                assert idx.reshape(-1)[a] == ul[j] + e0
                seen.append(int(a))
        assert np.all(np.diff(ul[:nl]) > 0) and np.all(ul[nl:] == -1)
    assert sorted(seen) == list(range(T * s.top_k))
