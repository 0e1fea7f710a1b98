"""Expert-parallel MoE layer over torch.distributed ranks (one process per GPU).

Rank r of W holds the routed experts of one contiguous id range [e0, e1) (an even split of
the E experts) and, on rank 0 only, the shared expert; every rank holds the router.  Per
call each rank
  1. routes the batch and takes its union over all E experts (replicated, identical on
     every rank: the router and its inputs are the same),
  2. keeps the union entries of its own range (coli_moe_union_restrict),
  3. runs the expert FFNs of those entries with the full routing weights
     (coli_moe_forward with n_experts = e1 - e0), and
  4. adds the ranks' partial outputs with one all-reduce of y (NCCL over NVLink between
     GPUs).
The pages' analogues are the all-resident multi-GPU host and cluster mode's one batched
request per layer (colibri README.zh-CN "实际成果"; the technical article's
"集群模式与开放问题清单").  The compute steps go through a backend object, by default
the CUDA library (`LibraryBackend`); the partition and the combine are this module's.
"""
from dataclasses import dataclass
from typing import Optional, Tuple

import torch
import torch.distributed as dist


def expert_range(n_experts: int, world: int, rank: int) -> Tuple[int, int]:
    """Contiguous, as even as possible: rank r holds [E r / W, E (r + 1) / W)."""
    if not 0 <= rank < world or n_experts < world:
        raise ValueError("need 0 <= rank < world <= n_experts")
    return n_experts * rank // world, n_experts * (rank + 1) // world


@dataclass
class Routing:
    idx: torch.Tensor        # [T][k] int32 (global expert ids)
    w: torch.Tensor          # [T][k] float32
    union_ids: torch.Tensor  # [E] int32
    n_union: torch.Tensor    # [1] int32
    offsets: torch.Tensor    # [E+1] int32
    assign: torch.Tensor     # [T*k] int32


class LibraryBackend:
    """The CUDA library's calls, on the current device."""

    def __init__(self, hidden, inter, n_experts, top_k, e0, e1, has_shared, T_max, device):
        from . import binding as B
        self.B = B
        self.full = B.make_dims(hidden, inter, n_experts, top_k, 1 if has_shared else 0)
        self.local = B.make_dims(hidden, inter, e1 - e0, top_k, 1 if has_shared else 0)
        self.bufs = B.LayerBuffers(self.full, T_max, device=device)
        El = e1 - e0
        i32 = dict(dtype=torch.int32, device=device)
        self.uid_l = torch.zeros(El, **i32)
        self.nu_l = torch.zeros(1, **i32)
        self.off_l = torch.zeros(El + 1, **i32)
        self.asg_l = torch.zeros(max(T_max * top_k, 1), **i32)
        self.ws_l = torch.zeros(B.coli_moe_workspace_bytes(self.local, T_max), dtype=torch.uint8, device=device)
        B.check(B.coli_moe_workspace_init(self.ws_l))

    def route(self, w_router, bias, x, T) -> Routing:
        b = self.bufs
        self.B.check(self.B.coli_moe_route_union(self.full, w_router, bias, x, T, b.idx, b.w, None, b.union_ids,
                                                 b.n_union, b.offsets, b.assign, b.ws), "coli_moe_route_union")
        return Routing(b.idx, b.w, b.union_ids, b.n_union, b.offsets, b.assign)

    def restrict(self, r: Routing, T, e0, e1) -> Routing:
        self.B.check(self.B.coli_moe_union_restrict(self.full, T, e0, e1, r.union_ids, r.n_union, r.offsets,
                                                    r.assign, self.uid_l, self.nu_l, self.off_l, self.asg_l),
                     "coli_moe_union_restrict")
        return Routing(r.idx, r.w, self.uid_l, self.nu_l, self.off_l, self.asg_l)

    def forward(self, weights, x, T, r: Routing, residual, y):
        self.B.check(self.B.coli_moe_forward(self.local, weights, x, T, r.idx, r.w, r.union_ids, r.n_union,
                                             r.offsets, r.assign, residual, y, self.ws_l), "coli_moe_forward")


class ExpertParallelLayer:
    """One MoE layer split over the ranks of `group` (or the default group)."""

    def __init__(self, n_experts: int, w_router, bias, local_weights, backend, group=None,
                 world: Optional[int] = None, rank: Optional[int] = None):
        self.group = group
        self.world = world if world is not None else dist.get_world_size(group)
        self.rank = rank if rank is not None else dist.get_rank(group)
        self.e0, self.e1 = expert_range(n_experts, self.world, self.rank)
        self.w_router, self.bias = w_router, bias
        self.weights = local_weights   # the rank's experts e0..e1-1 (and the shared one on rank 0)
        self.backend = backend

    def forward(self, x: torch.Tensor, T: int, residual: Optional[torch.Tensor] = None) -> torch.Tensor:
        r = self.backend.route(self.w_router, self.bias, x, T)
        rl = self.backend.restrict(r, T, self.e0, self.e1)
        y = torch.empty(T, x.shape[-1], dtype=torch.float32, device=x.device)
        # the residual enters once, on rank 0 (like the shared expert)
        self.backend.forward(self.weights, x, T, rl, residual if self.rank == 0 else None, y)
        if self.world > 1:
            dist.all_reduce(y, op=dist.ReduceOp.SUM, group=self.group)
        return y
