"""Owner-partitioned Muon step across data-parallel ranks.

Each matrix has one owner rank, chosen by a longest-processing-time-first
partition of the Newton-Schulz cost 3 m^2 n per step (the DMuon quick start,
"刚才发生了什么": each projection is assigned to a single owner by a balanced
LPT partition; the blog's "参数分片减少 N-S 计算量": each rank runs N-S only
on its share).  One step:

1. the gradients are reduced to their owners (sum, then divided by the
   number of ranks: the data-parallel mean), all reductions in flight at
   once;
2. every owner runs one batched Muon update over the matrices it owns (one
   launch per stage on the GPU) -- only owners keep momentum buffers;
3. every updated matrix is broadcast from its owner.

The collectives go through ``torch.distributed`` (NCCL on GPUs, gloo on
CPUs); the update itself is ``dmuon_muon_step_batched`` unless a step
function is given (the CPU tests pass one).
"""
from __future__ import annotations

import heapq
from typing import Callable, List, Optional, Sequence

import torch
import torch.distributed as dist


def ns_cost(rows: int, cols: int, steps: int = 5) -> float:
    """Useful Newton-Schulz FLOPs of one matrix: steps * 3 m^2 n."""
    m, n = min(rows, cols), max(rows, cols)
    return float(steps) * 3.0 * m * m * n


def lpt_partition(costs: Sequence[float], world: int) -> List[int]:
    """Owner rank of each item: items in decreasing cost order, each to the
    currently least loaded rank (ties to the lower rank, then the lower item
    index, so every rank computes the same assignment)."""
    if world < 1:
        raise ValueError("world must be >= 1")
    order = sorted(range(len(costs)), key=lambda i: (-costs[i], i))
    heap = [(0.0, r) for r in range(world)]
    owner = [0] * len(costs)
    for i in order:
        load, r = heapq.heappop(heap)
        owner[i] = r
        heapq.heappush(heap, (load + costs[i], r))
    return owner


def imbalance(costs: Sequence[float], owner: Sequence[int], world: int) -> float:
    """max load / mean load - 1."""
    loads = [0.0] * world
    for c, r in zip(costs, owner):
        loads[r] += c
    mean = sum(loads) / world
    return max(loads) / mean - 1.0 if mean > 0 else 0.0


StepFn = Callable[..., None]


def _default_step(params, grads, bufs, **kw) -> None:
    from . import dmuon_muon_step_batched
    dmuon_muon_step_batched(params, grads, bufs, **kw)


class OwnerPartitionedMuon:
    """Muon over data-parallel ranks with one owner per matrix.

    ``params`` are the full replicated weights (same on every rank).  Each
    rank allocates momentum buffers only for the matrices it owns.
    """

    def __init__(self, params: Sequence[torch.Tensor], group=None, ns_steps: int = 5,
                 step_fn: Optional[StepFn] = None):
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        self.params = list(params)
        self.ns_steps = ns_steps
        costs = [ns_cost(p.shape[0], p.shape[1], ns_steps) for p in self.params]
        self.owner = lpt_partition(costs, self.world)
        self.owned = [i for i, r in enumerate(self.owner) if r == self.rank]
        self.bufs = {i: torch.zeros(self.params[i].shape, dtype=torch.float32,
                                    device=self.params[i].device) for i in self.owned}
        self.step_fn = step_fn or _default_step
        self.imbalance = imbalance(costs, self.owner, self.world)

    def _global_rank(self, r: int) -> int:
        return r if self.group is None else dist.get_global_rank(self.group, r)

    @torch.no_grad()
    def step(self, grads: Sequence[Optional[torch.Tensor]], lr: float = 0.02,
             momentum: float = 0.95, nesterov: bool = True, weight_decay: float = 0.0) -> None:
        """One step.  ``grads`` are this rank's local gradients (None for a
        parameter without gradient on every rank); they are overwritten by
        the reduction on the owner."""
        # 1. reduce every gradient to its owner, all in flight at once
        work = []
        for i, g in enumerate(grads):
            if g is None:
                continue
            work.append(dist.reduce(g, dst=self._global_rank(self.owner[i]), op=dist.ReduceOp.SUM,
                                    group=self.group, async_op=True))
        for w in work:
            w.wait()
        # 2. owners update their matrices in one batched call
        ps, gs, bs = [], [], []
        for i in self.owned:
            if grads[i] is None:
                continue
            g = grads[i]
            if self.world > 1:
                g.div_(self.world)
            ps.append(self.params[i])
            gs.append(g)
            bs.append(self.bufs[i])
        if ps:
            self.step_fn(ps, gs, bs, lr=lr, momentum=momentum, nesterov=nesterov,
                         weight_decay=weight_decay, ns_steps=self.ns_steps)
        # 3. broadcast every updated matrix from its owner
        work = []
        for i, g in enumerate(grads):
            if g is None:
                continue
            work.append(dist.broadcast(self.params[i], src=self._global_rank(self.owner[i]),
                                       group=self.group, async_op=True))
        for w in work:
            w.wait()
