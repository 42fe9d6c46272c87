"""Data-parallel Muon over several ranks: whole-matrix ownership + exchange.

Newton-Schulz needs whole matrices ("Muon 优化器完全拆解…", section
"分布式工程": Distributed Muon gathers the full matrix before orthogonalising;
DeepSeek-V4 assigns matrices to buckets with a knapsack). Here every rank
holds the full weights and gradients (data parallelism after the gradient
all-reduce), and:

1. matrices are assigned to ranks whole, largest first, each to the rank with
   the least Newton-Schulz work so far (a greedy knapsack on the FLOP count);
2. each rank runs the single-GPU step (muon_step_b200.MuonPlan) over the
   matrices it owns: momentum buffers of other ranks' matrices are not
   touched and may be omitted (ZeRO-1 style optimizer-state sharding);
3. every owner broadcasts its updated weights as one packed buffer (NCCL over
   NVLink between GPUs), so all ranks end the step with identical weights.

One process per GPU, torch.distributed for the plumbing.
"""

from __future__ import annotations

from typing import Callable, Optional, Sequence

import torch
import torch.distributed as dist


def ns_cost(shape) -> float:
    """Newton-Schulz FLOPs of one step on an n x m matrix, 4 r^2 c + 2 r^3."""
    n, m = shape
    r, c = min(n, m), max(n, m)
    return 4.0 * r * r * c + 2.0 * r ** 3


def partition(shapes: Sequence, world: int) -> list:
    """Owner rank of each matrix: largest first, to the least-loaded rank
    (ties to the lower rank). Deterministic, so every rank computes the same."""
    if world < 1:
        raise ValueError("world must be >= 1")
    order = sorted(range(len(shapes)), key=lambda k: (-ns_cost(shapes[k]), k))
    load = [0.0] * world
    owner = [0] * len(shapes)
    for k in order:
        r = min(range(world), key=lambda i: (load[i], i))
        owner[k] = r
        load[r] += ns_cost(shapes[k])
    return owner


class DistributedMuon:
    """Muon step over matrices shared by every rank of ``group``.

    params: list of (W, G, M) per matrix, identical shapes and order on every
    rank; M may be None on ranks that do not own the matrix. ``compute``
    replaces the per-rank single-GPU step (a callable taking the owned
    indices and the hyper-parameters), e.g. for tests on CPU ranks.
    """

    def __init__(self, params: Sequence, group=None, precision="bf16", schedule=None,
                 eps=None, compute: Optional[Callable] = None):
        self.group = group
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)
        self.params = list(params)
        shapes = [tuple(p[0].shape) for p in self.params]
        self.owner = partition(shapes, self.world)
        self.owned = [[k for k, o in enumerate(self.owner) if o == r] for r in range(self.world)]
        mine = self.owned[self.rank]
        for k in mine:
            if self.params[k][2] is None:
                raise ValueError(f"rank {self.rank} owns matrix {k} but has no momentum buffer")
        if compute is None:
            from . import MuonPlan

            plan = MuonPlan([self.params[k][:3] for k in mine], precision, schedule, eps) if mine else None
            ws = plan.alloc_workspace() if plan is not None else None

            def compute(owned, hyper):
                if plan is not None:
                    plan.execute(ws, **hyper)

            self._plan, self._ws = plan, ws
        self._compute = compute
        W0 = self.params[0][0]
        self._bufs = [torch.empty(sum(self.params[k][0].numel() for k in self.owned[r]),
                                  dtype=W0.dtype, device=W0.device) for r in range(self.world)]

    def _src(self, r):
        return dist.get_global_rank(self.group, r) if self.group is not None else r

    def step(self, lr=0.02, momentum=0.95, weight_decay=0.1, gamma=0.2, nesterov=True):
        hyper = dict(lr=lr, momentum=momentum, weight_decay=weight_decay, gamma=gamma,
                     nesterov=nesterov)
        mine = self.owned[self.rank]
        self._compute(mine, hyper)
        # pack this rank's updated weights
        buf, off = self._bufs[self.rank], 0
        for k in mine:
            W = self.params[k][0]
            buf[off:off + W.numel()].copy_(W.reshape(-1))
            off += W.numel()
        # every owner broadcasts, in rank order (the same sequence on every rank)
        for r in range(self.world):
            if self._bufs[r].numel():
                dist.broadcast(self._bufs[r], src=self._src(r), group=self.group)
        # unpack the other owners' weights
        for r in range(self.world):
            if r == self.rank:
                continue
            off = 0
            for k in self.owned[r]:
                W = self.params[k][0]
                W.copy_(self._bufs[r][off:off + W.numel()].view_as(W))
                off += W.numel()
