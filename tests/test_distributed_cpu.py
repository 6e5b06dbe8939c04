"""Owner-partitioned Muon over data-parallel ranks, on CPU (gloo, 2-3 ranks).

The per-owner update is the fp64 oracle (injected as the step function, with
the oracle's rank mean: an fp32 sum in rank order, then one division), so
these tests check the partition, the transfer of every rank's gradient to its
owner in rank order, the owners' batched step and the broadcast: the result
on every rank must equal one step of the oracle on the rank mean, bit for
bit.  The gradients are random fp32 values whose sums round, so a different
summation order or a reduction in another precision would show.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from newton_schulz_09_b200 import distributed as dmd
from newton_schulz_09_b200 import synthetic

SHAPES = [(48, 96), (96, 48), (64, 64), (32, 128), (24, 40), (128, 32), (16, 16)]
HP = dict(lr=0.02, momentum=0.95, nesterov=True, weight_decay=0.01)


def oracle_step_fn(ps, rank_grads, bs, *, lr, momentum, nesterov, weight_decay, ns_steps):
    for k, (p, b) in enumerate(zip(ps, bs)):
        g = oracle.rank_mean([rank_grads[r][k].numpy() for r in range(len(rank_grads))])
        buf_new, X, W_new = oracle.muon_step(p.numpy(), g, b.numpy(), lr=lr, momentum=momentum,
                                             nesterov=nesterov, weight_decay=weight_decay,
                                             ns_steps=ns_steps)
        b.copy_(torch.from_numpy(buf_new))
        p.copy_(torch.from_numpy(W_new.astype(np.float32)))


def _params():
    gen = torch.Generator().manual_seed(5)
    return [torch.randn(s, generator=gen) * 0.02 for s in SHAPES]


def _grads(rank, step):
    # random fp32 values of varied magnitude: their sums over ranks round, so
    # the mean depends on the order and precision of the sum
    gen = torch.Generator().manual_seed(1000 * step + rank)
    gs = [torch.randn(s, generator=gen) * 10.0 ** (-3 + rank) for s in SHAPES]
    gs[4] = None if step == 1 else gs[4]          # no gradient for one matrix on step 1
    return gs


def _worker(rank, world, port, out_dir):
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world)
    try:
        params = _params()
        opt = dmd.OwnerPartitionedMuon(params, ns_steps=3, step_fn=oracle_step_fn)
        untouched = True
        for step in range(2):
            gs = _grads(rank, step)
            g0 = [None if g is None else g.clone() for g in gs]
            opt.step(gs, **HP)
            untouched = untouched and all(a is None or torch.equal(a, b) for a, b in zip(gs, g0))
        torch.save({"params": [p.clone() for p in params], "owner": opt.owner, "untouched": untouched,
                    "owned": opt.owned, "bufs": {i: b.clone() for i, b in opt.bufs.items()}},
                   os.path.join(out_dir, f"rank{rank}.pt"))
    finally:
        dist.destroy_process_group()


def _resume_worker(rank, world, port, out_dir):
    """Two steps in one go, or one step, a checkpoint, a fresh optimizer
    restored from it, and the second step: the results must be identical."""
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world)
    try:
        straight = _params()
        opt = dmd.OwnerPartitionedMuon(straight, ns_steps=3, step_fn=oracle_step_fn)
        for step in range(2):
            opt.step(_grads(rank, step), **HP)
        resumed = _params()
        opt1 = dmd.OwnerPartitionedMuon(resumed, ns_steps=3, step_fn=oracle_step_fn)
        opt1.step(_grads(rank, 0), **HP)
        saved = opt1.state_dict()
        opt2 = dmd.OwnerPartitionedMuon(resumed, ns_steps=3, step_fn=oracle_step_fn)
        opt2.load_state_dict(saved)
        opt2.step(_grads(rank, 1), **HP)
        same = all(torch.equal(a, b) for a, b in zip(straight, resumed))
        same = same and all(torch.equal(opt.bufs[i], opt2.bufs[i]) for i in opt.bufs)
        torch.save({"same": same}, os.path.join(out_dir, f"resume{rank}.pt"))
    finally:
        dist.destroy_process_group()


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def test_lpt_partition_is_deterministic_and_balanced():
    wl = synthetic.workload("llama8b")
    costs = [dmd.ns_cost(s.rows, s.cols) for s in wl.specs]
    for world in (2, 4, 8):
        owner = dmd.lpt_partition(costs, world)
        assert owner == dmd.lpt_partition(costs, world)
        assert set(owner) == set(range(world))
        assert dmd.imbalance(costs, owner, world) < 0.02
    # one dominant item: it sits alone on its rank
    owner = dmd.lpt_partition([100.0, 1.0, 1.0, 1.0], 2)
    assert owner[0] != owner[1] and owner[1] == owner[2] == owner[3]
    assert dmd.lpt_partition([3.0, 2.0], 1) == [0, 0]
    with pytest.raises(ValueError):
        dmd.lpt_partition([1.0], 0)


def test_owner_chunks_and_global_schedule():
    owner = [0, 1, 0, 0, 1, 2, 0, 0]
    numel = [10, 5, 10, 10, 5, 7, 10, 10]
    ch = dmd.owner_chunks(owner, numel, 3, chunks_per_owner=2)
    # each owner's matrices, in index order, cut into consecutive chunks
    for r in range(3):
        assert sum(ch[r], []) == [i for i, o in enumerate(owner) if o == r]
        assert 1 <= len(ch[r]) <= 2
    assert ch[0] == [[0, 2, 3], [6, 7]]
    sched = dmd.global_schedule(ch)
    # chunk 0 of every owner, then chunk 1 of those that have one
    assert sched[:3] == [(0, 0), (1, 0), (2, 0)]
    assert sorted(sched) == sorted((r, c) for r in range(3) for c in range(len(ch[r])))
    assert dmd.global_schedule([[], [[1]]]) == [(1, 0)]


@pytest.mark.parametrize("world", [2, 3])
def test_ranks_match_one_step_on_averaged_gradients(scratch_dir, world):
    mp.start_processes(_worker, args=(world, _free_port(), str(scratch_dir)), nprocs=world,
                       start_method="spawn", join=True)
    res = [torch.load(scratch_dir / f"rank{r}.pt") for r in range(world)]
    # every rank holds identical weights after the broadcasts
    for r in range(1, world):
        for a, b in zip(res[0]["params"], res[r]["params"]):
            assert torch.equal(a, b)
    # every matrix has exactly one owner, and only owners keep buffers
    assert sorted(sum((res[r]["owned"] for r in range(world)), [])) == list(range(len(SHAPES)))
    # the callers' gradients are only read
    assert all(res[r]["untouched"] for r in range(world))
    # reference: two oracle steps on the oracle's rank mean (fp32 sum in rank
    # order, then one division)
    W = [p.numpy().copy() for p in _params()]
    bufs = [np.zeros(s, np.float32) for s in SHAPES]
    for step in range(2):
        gr = [_grads(r, step) for r in range(world)]
        for i in range(len(SHAPES)):
            if gr[0][i] is None:
                continue
            gm = oracle.rank_mean([g[i].numpy() for g in gr])
            # the gradients are not exactly summable: another order of the
            # fp32 sum, or a sum in fp64, gives a different mean somewhere
            wide = (sum(g[i].numpy().astype(np.float64) for g in gr) / world).astype(np.float32)
            if world > 2:
                assert not np.array_equal(gm, wide)
            bufs[i], _, Wn = oracle.muon_step(W[i], gm, bufs[i], ns_steps=3, **HP)
            W[i] = Wn.astype(np.float32)
    for i in range(len(SHAPES)):
        got = res[0]["params"][i].numpy()
        assert np.array_equal(got, W[i]), i
        owner = res[0]["owner"][i]
        assert np.array_equal(res[owner]["bufs"][i].numpy(), bufs[i])


def test_checkpoint_and_resume(scratch_dir):
    world = 2
    mp.start_processes(_resume_worker, args=(world, _free_port(), str(scratch_dir)), nprocs=world,
                       start_method="spawn", join=True)
    for r in range(world):
        assert torch.load(scratch_dir / f"resume{r}.pt")["same"]


def test_load_state_dict_checks_the_partition():
    opt = dmd.OwnerPartitionedMuon.__new__(dmd.OwnerPartitionedMuon)
    opt.owner = [0, 1, 0]
    opt.bufs = {0: torch.zeros(2), 2: torch.zeros(3)}
    opt.ns_steps = 5
    with pytest.raises(ValueError):
        opt.load_state_dict({"owner": [1, 0, 0], "ns_steps": 5, "bufs": {}})
    with pytest.raises(ValueError):
        opt.load_state_dict({"owner": [0, 1, 0], "ns_steps": 5, "bufs": {0: torch.ones(2)}})
    opt.load_state_dict({"owner": [0, 1, 0], "ns_steps": 3, "bufs": {0: torch.ones(2), 2: torch.ones(3)}})
    assert torch.equal(opt.bufs[2], torch.ones(3)) and opt.ns_steps == 3
