"""The owner-partitioned step on the GPU through NCCL with one rank: the
reduction and broadcast are no-ops, so the result must equal a direct
batched step bit for bit (needs a B200)."""
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

import oracle
from newton_schulz_09_b200 import distributed as dmd
from tests.gpu_helpers import check_bf16_weights, host

pytestmark = pytest.mark.gpu


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def test_single_rank_nccl_matches_direct_step(cuda_lib):
    dm = cuda_lib
    dev = torch.device("cuda:0")
    gen = torch.Generator(device=dev).manual_seed(3)
    shapes = [(512, 1536), (1536, 512), (256, 256)]
    pa = [(torch.randn(s, generator=gen, device=dev) * 0.02).to(torch.bfloat16) for s in shapes]
    pb = [p.clone() for p in pa]
    grads = [(torch.randn(s, generator=gen, device=dev) * 1e-3).to(torch.bfloat16) for s in shapes]
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0, world_size=1)
    try:
        W0 = [host(p) for p in pa]
        opt = dmd.OwnerPartitionedMuon(pa)
        assert opt.owned == [0, 1, 2]
        gcopy = [g.clone() for g in grads]
        opt.step(gcopy, lr=0.02, weight_decay=0.01)
        bufs = [torch.zeros(s, dtype=torch.float32, device=dev) for s in shapes]
        dm.dmuon_muon_step_batched(pb, grads, bufs, lr=0.02, weight_decay=0.01)
        torch.cuda.synchronize()
        for a, b in zip(pa, pb):
            assert torch.equal(a, b)
        for i in range(3):
            assert torch.equal(opt.bufs[i], bufs[i])
        # the gradients are only read, and the result is the oracle's step on
        # the rank mean (here of one rank)
        for g, h in zip(gcopy, grads):
            assert torch.equal(g, h)
        for i, s in enumerate(shapes):
            gm = oracle.rank_mean([host(grads[i])])
            buf_ref, X, W_ref = oracle.muon_step(W0[i], gm, np.zeros(s, np.float32), lr=0.02,
                                                 momentum=0.95, nesterov=True, weight_decay=0.01,
                                                 ns_steps=5)
            assert np.array_equal(host(opt.bufs[i]).view(np.uint32), buf_ref.view(np.uint32))
            check_bf16_weights(host(pa[i]), W_ref, X, 0.02, f"owner step W {s}")
    finally:
        dist.destroy_process_group()


def test_single_rank_peer_mode_matches_direct_step(cuda_lib):
    """Gradients in symmetric memory, read by the owner's fused step: with one
    rank the result equals a direct batched step bit for bit."""
    dm = cuda_lib
    dev = torch.device("cuda:0")
    gen = torch.Generator(device=dev).manual_seed(4)
    shapes = [(512, 1536), (1536, 512), (256, 256), (130, 72)]
    pa = [(torch.randn(s, generator=gen, device=dev) * 0.02).to(torch.bfloat16) for s in shapes]
    pb = [p.clone() for p in pa]
    grads = [(torch.randn(s, generator=gen, device=dev) * 1e-3).to(torch.bfloat16) for s in shapes]
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0, world_size=1)
    try:
        opt = dmd.OwnerPartitionedMuon(pa, grad_exchange="peer")
        for g, view in zip(grads, opt.grads):
            view.copy_(g)
        opt.step_peer(lr=0.02, weight_decay=0.01)
        bufs = [torch.zeros(s, dtype=torch.float32, device=dev) for s in shapes]
        dm.dmuon_muon_step_batched(pb, grads, bufs, lr=0.02, weight_decay=0.01)
        torch.cuda.synchronize()
        for a, b in zip(pa, pb):
            assert torch.equal(a, b)
        for i in range(len(shapes)):
            assert torch.equal(opt.bufs[i], bufs[i])
    finally:
        dist.destroy_process_group()
