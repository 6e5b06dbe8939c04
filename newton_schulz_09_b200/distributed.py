"""Owner-partitioned Muon step across data-parallel ranks.

Each matrix has one owner rank, chosen by a longest-processing-time-first
partition of the Newton-Schulz cost 3 m^2 n per step (the DMuon quick start,
"刚才发生了什么": each projection is assigned to a single owner by a balanced
LPT partition; the blog's "参数分片减少 N-S 计算量": each rank runs N-S only
on its share).  One step:

1. every rank's gradient of a matrix reaches the matrix's owner unreduced
   (point-to-point sends, one batch per chunk of the schedule below, all
   batches issued at once); the caller's gradients are only read;
2. every owner updates the matrices it owns in a few chunks, one batched
   call each (only owners keep momentum buffers).  The call is
   ``dmuon_muon_step_batched_reduce``: its prologue forms the data-parallel
   mean of the ranks' gradients itself, an fp32 sum in rank order and one
   fp32 division by the number of ranks, so the mean does not depend on how
   a collective happens to order or round its sums.  A chunk waits only for
   its own transfers, so later transfers run while earlier chunks compute;
3. every updated matrix is broadcast from its owner as soon as its chunk is
   done, while later chunks compute.

All ranks issue the same communication in the same order: the transfer
batches, then the broadcasts, chunk by chunk in one global schedule that
interleaves the owners.  It goes through ``torch.distributed`` (NCCL on
GPUs, gloo on CPUs), whose waits are stream-ordered on GPUs.  The owner's
update is the library's unless a function is given (the CPU tests pass the
oracle).

Memory: an owner keeps one receive buffer per other rank for each matrix it
owns, (world - 1) times its share of the gradients, allocated on the first
step and reused.
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


def _default_reduce_step(params, rank_grads, bufs, **kw) -> None:
    """The owner's update on every rank's gradients (``rank_grads[r][k]``)."""
    from . import dmuon_muon_step_batched_reduce
    dmuon_muon_step_batched_reduce(params, rank_grads, bufs, **kw)


def owner_chunks(owner: Sequence[int], numel: Sequence[int], world: int,
                 chunks_per_owner: int = 4) -> List[List[List[int]]]:
    """Per owner rank, its matrices (in index order) cut into at most
    ``chunks_per_owner`` consecutive chunks of about equal element count."""
    out: List[List[List[int]]] = []
    for r in range(world):
        mine = [i for i, o in enumerate(owner) if o == r]
        total = sum(numel[i] for i in mine)
        target = total / max(1, chunks_per_owner)
        chunks: List[List[int]] = []
        cur: List[int] = []
        acc = 0
        for i in mine:
            cur.append(i)
            acc += numel[i]
            if acc >= target and len(chunks) + 1 < chunks_per_owner:
                chunks.append(cur)
                cur, acc = [], 0
        if cur:
            chunks.append(cur)
        out.append(chunks)
    return out


def global_schedule(chunks: Sequence[Sequence[Sequence[int]]]) -> List[tuple]:
    """(owner, chunk index) pairs, chunk 0 of every owner first, then chunk 1, ..."""
    depth = max((len(c) for c in chunks), default=0)
    return [(r, c) for c in range(depth) for r in range(len(chunks)) if c < len(chunks[r])]


class OwnerPartitionedMuon:
    """Muon over data-parallel ranks with one owner per matrix.

    ``params`` are the full replicated weights (same on every rank).  Each
    rank allocates momentum buffers only for the matrices it owns.

    ``grad_exchange``: "nccl" (default) sends every rank's gradient to the
    owner, whose update averages them.  "peer" keeps the gradients in
    symmetric memory (``self.grads``, one view per parameter in the parameter's dtype, which
    the caller fills): after a stream-ordered barrier each owner reads every
    rank's gradient of the matrices it owns straight from peer memory inside
    its update (``dmuon_muon_step_batched_reduce``), so no reduced copy is
    written; the updated weights are then broadcast as in the NCCL mode.

    ``step_fn(params, rank_grads, bufs, lr=, momentum=, nesterov=,
    weight_decay=, ns_steps=)`` replaces the owner's update (the CPU tests
    pass the oracle); ``rank_grads[r][k]`` is rank r's gradient of
    ``params[k]``.
    """

    def __init__(self, params: Sequence[torch.Tensor], group=None, ns_steps: int = 5,
                 step_fn: Optional[StepFn] = None, chunks_per_owner: int = 4,
                 grad_exchange: str = "nccl"):
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
        self.step_fn = step_fn or _default_reduce_step
        self._recv: dict = {}           # (matrix, rank) -> receive buffer on the owner
        self.imbalance = imbalance(costs, self.owner, self.world)
        self.chunks = owner_chunks(self.owner, [p.numel() for p in self.params], self.world,
                                   chunks_per_owner)
        self.schedule = global_schedule(self.chunks)
        if grad_exchange not in ("nccl", "peer"):
            raise ValueError("grad_exchange must be 'nccl' or 'peer'")
        self.grad_exchange = grad_exchange
        self.grads: Optional[List[torch.Tensor]] = None
        if grad_exchange == "peer":
            self._setup_peer()

    def _setup_peer(self) -> None:
        """One symmetric buffer per gradient dtype holding every parameter's
        gradient (16-byte aligned offsets), and views of every rank's copy."""
        import torch.distributed._symmetric_memory as symm
        dev = self.params[0].device
        if dev.type != "cuda":
            raise ValueError("grad_exchange='peer' needs CUDA parameters")
        group = self.group if self.group is not None else dist.group.WORLD
        self.grads = [None] * len(self.params)
        self._peer: dict = {}
        self._handles = []
        by_dtype: dict = {}
        for i, p in enumerate(self.params):
            by_dtype.setdefault(p.dtype, []).append(i)
        for dt in sorted(by_dtype, key=str):            # the same order on every rank
            idx = by_dtype[dt]
            align = 16 // torch.empty((), dtype=dt).element_size()
            offs, total = [], 0
            for i in idx:
                offs.append(total)
                total += -(-self.params[i].numel() // align) * align
            buf = symm.empty(total, dtype=dt, device=dev)
            hdl = symm.rendezvous(buf, group)
            self._handles.append((buf, hdl))
            for i, off in zip(idx, offs):
                n, shape = self.params[i].numel(), self.params[i].shape
                self.grads[i] = buf[off:off + n].view(shape)
                self._peer[i] = [hdl.get_buffer(r, (n,), dt, off).view(shape) for r in range(self.world)]

    def state_dict(self) -> dict:
        """This rank's optimizer state: the momentum buffers of the matrices
        it owns (by parameter index) and the partition they belong to."""
        return {"owner": list(self.owner), "ns_steps": self.ns_steps,
                "bufs": {i: b.detach().clone() for i, b in self.bufs.items()}}

    def load_state_dict(self, state: dict) -> None:
        """Restores buffers saved by ``state_dict`` on the same rank of a job
        with the same parameters and number of ranks (so the same partition)."""
        if list(state["owner"]) != self.owner:
            raise ValueError("the saved state belongs to another partition of the parameters")
        if set(state["bufs"]) != set(self.bufs):
            raise ValueError("the saved buffers are not this rank's")
        for i, b in state["bufs"].items():
            self.bufs[i].copy_(b)
        self.ns_steps = int(state["ns_steps"])

    def _global_rank(self, r: int) -> int:
        return r if self.group is None else dist.get_global_rank(self.group, r)

    @torch.no_grad()
    def step_peer(self, lr: float = 0.02, momentum: float = 0.95, nesterov: bool = True,
                  weight_decay: float = 0.0) -> None:
        """One step of the "peer" mode: every rank has written its gradients
        into ``self.grads`` on its current stream.  Enqueues only."""
        from . import dmuon_muon_step_batched_reduce
        if self.grad_exchange != "peer":
            raise RuntimeError("step_peer needs grad_exchange='peer'")
        # Stream-ordered barrier: a collective completes only once every rank's
        # stream has reached it, i.e. once every rank's gradients are written.
        flag = torch.zeros(1, device=self.params[0].device)
        dist.all_reduce(flag, group=self.group)
        bcast = []
        for r, c in self.schedule:
            idx = self.chunks[r][c]
            if r == self.rank:
                dmuon_muon_step_batched_reduce(
                    [self.params[i] for i in idx],
                    [[self._peer[i][q] for i in idx] for q in range(self.world)],
                    [self.bufs[i] for i in idx], lr=lr, momentum=momentum, nesterov=nesterov,
                    weight_decay=weight_decay, ns_steps=self.ns_steps)
            for i in idx:
                bcast.append(dist.broadcast(self.params[i], src=self._global_rank(r), group=self.group,
                                            async_op=True))
        for w in bcast:
            w.wait()

    def _recv_buffer(self, i: int, q: int, like: torch.Tensor) -> torch.Tensor:
        key = (i, q)
        b = self._recv.get(key)
        if b is None or b.shape != like.shape or b.dtype != like.dtype or b.device != like.device:
            b = torch.empty_like(like, memory_format=torch.contiguous_format)
            self._recv[key] = b
        return b

    @torch.no_grad()
    def step(self, grads: Sequence[Optional[torch.Tensor]], lr: float = 0.02,
             momentum: float = 0.95, nesterov: bool = True, weight_decay: float = 0.0) -> None:
        """One step.  ``grads`` are this rank's local gradients (None for a
        parameter without gradient on every rank); they are read, not
        modified.  On GPUs the call only enqueues work (the collectives'
        waits are stream-ordered); the parameters are final once the current
        stream reaches the end of the step."""
        # 1. per chunk of the schedule, one batch of point-to-point transfers:
        # every other rank's gradient of the chunk's matrices to their owner
        pending = {}
        for r, c in self.schedule:
            idx = [i for i in self.chunks[r][c] if grads[i] is not None]
            if not idx or self.world == 1:
                continue
            ops = []
            if r == self.rank:
                for i in idx:
                    for q in range(self.world):
                        if q != self.rank:
                            ops.append(dist.P2POp(dist.irecv, self._recv_buffer(i, q, grads[i]),
                                                  self._global_rank(q), self.group))
            else:
                for i in idx:
                    ops.append(dist.P2POp(dist.isend, grads[i].contiguous(), self._global_rank(r),
                                          self.group))
            pending[(r, c)] = dist.batch_isend_irecv(ops)
        # 2.-3. chunk by chunk in the global schedule: the owner updates its
        # chunk on every rank's gradients once they have arrived, then every
        # rank takes part in the chunk's broadcasts
        bcast = []
        for r, c in self.schedule:
            idx = [i for i in self.chunks[r][c] if grads[i] is not None]
            if not idx:
                continue
            if r == self.rank:
                for w in pending.get((r, c), []):
                    w.wait()
                rank_grads = [[grads[i] if q == self.rank else self._recv[(i, q)] for i in idx]
                              for q in range(self.world)]
                self.step_fn([self.params[i] for i in idx], rank_grads, [self.bufs[i] for i in idx],
                             lr=lr, momentum=momentum, nesterov=nesterov, weight_decay=weight_decay,
                             ns_steps=self.ns_steps)
            for i in idx:
                bcast.append(dist.broadcast(self.params[i], src=self._global_rank(r), group=self.group,
                                            async_op=True))
        for (r, c), works in pending.items():
            if r != self.rank:
                for w in works:
                    w.wait()
        for w in bcast:
            w.wait()
