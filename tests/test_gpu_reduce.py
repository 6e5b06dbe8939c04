"""The owner's step with the data-parallel gradient reduction fused into the
update (needs a B200).  The ranks are emulated by separate buffers on this
GPU: the kernel reads every rank's buffer directly in any case, whether the
memory is local or mapped from a peer.  Momentum buffers must match the
oracle on the rank mean bit for bit; the weights follow the usual tolerance."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from tests.gpu_helpers import TOL_BF16, TOL_F32, check_bf16_weights, check_rel, host

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
SHAPES = [((384, 1024), torch.bfloat16), ((1200, 264), torch.bfloat16), ((200, 72), torch.float32),
          ((130, 67), torch.bfloat16), ((4096, 1024), torch.bfloat16)]
HP = dict(lr=0.02, momentum=0.95, nesterov=True, weight_decay=0.01, ns_steps=5)


def _rand(shape, dtype, seed, std=1.0):
    g = torch.Generator(device=DEV)
    g.manual_seed(seed)
    return (torch.randn(shape, generator=g, device=DEV) * std).to(dtype)


@pytest.mark.parametrize("world", [2, 3, 8])
def test_rank_mean_step_against_oracle(cuda_lib, world):
    dm = cuda_lib
    params = [_rand(s, d, 10 + i, 0.02) for i, (s, d) in enumerate(SHAPES)]
    bufs = [_rand(s, torch.float32, 30 + i, 1e-3) for i, (s, d) in enumerate(SHAPES)]
    W0 = [host(p) for p in params]
    b0 = [host(b) for b in bufs]
    rank_grads = [[_rand(s, d, 1000 * r + i, 1e-3) for i, (s, d) in enumerate(SHAPES)] for r in range(world)]
    rank_grads_host = [[host(g) for g in gs] for gs in rank_grads]
    dm.dmuon_muon_step_batched_reduce(params, rank_grads, bufs, **HP)
    torch.cuda.synchronize()
    assert dm.dmuon_device_status() == 0
    for i, (s, d) in enumerate(SHAPES):
        gm = oracle.rank_mean([rank_grads_host[r][i] for r in range(world)])
        buf_ref, X, W_ref = oracle.muon_step(W0[i], gm, b0[i], **HP)
        assert np.array_equal(host(bufs[i]).view(np.uint32), buf_ref.view(np.uint32)), (world, i)
        if d == torch.bfloat16:
            check_bf16_weights(host(params[i]), W_ref, X, HP["lr"], f"W {s} world {world}")
        else:
            check_rel(host(params[i]) - W0[i], W_ref - W0[i], TOL_F32, f"dW {s} world {world}")


def test_equals_the_plain_step_on_the_mean(cuda_lib):
    """fp32 gradients: the mean formed by torch in the same order (sum in
    rank order, then one division) and passed to the plain entry point gives
    the same bits."""
    dm = cuda_lib
    world = 4
    shapes = [(512, 1536), (1536, 512), (96, 200)]
    params = [_rand(s, torch.bfloat16, 50 + i, 0.02) for i, s in enumerate(shapes)]
    bufs = [torch.zeros(s, dtype=torch.float32, device=DEV) for s in shapes]
    ref_p, ref_b = [p.clone() for p in params], [b.clone() for b in bufs]
    rank_grads = [[_rand(s, torch.float32, 70 + 10 * r + i, 1e-3) for i, s in enumerate(shapes)]
                  for r in range(world)]
    mean = []
    for i in range(len(shapes)):
        acc = rank_grads[0][i].clone()
        for r in range(1, world):
            acc = acc + rank_grads[r][i]
        mean.append(acc / world)
    dm.dmuon_muon_step_batched_reduce(params, rank_grads, bufs, **HP)
    dm.dmuon_muon_step_batched_opts(ref_p, mean, ref_b, **HP)
    torch.cuda.synchronize()
    for i in range(len(shapes)):
        assert torch.equal(bufs[i], ref_b[i]), i
        assert torch.equal(params[i], ref_p[i]), i


def test_skips_and_rejects(cuda_lib):
    dm = cuda_lib
    s = (256, 512)
    p = _rand(s, torch.bfloat16, 1, 0.02)
    p0 = p.clone()
    b = torch.zeros(s, dtype=torch.float32, device=DEV)
    # no gradient on any rank: the matrix is skipped
    dm.dmuon_muon_step_batched_reduce([p], [[None], [None]], [b], **HP)
    torch.cuda.synchronize()
    assert torch.equal(p, p0)
    # a gradient on some ranks only is refused, by the binding and by the C ABI
    g = _rand(s, torch.bfloat16, 2, 1e-3)
    with pytest.raises(ValueError):
        dm.dmuon_muon_step_batched_reduce([p], [[g], [None]], [b], **HP)
    lib = dm.load_library()
    o = dm.DmuonStepOptions()
    lib.dmuon_step_options_default(ctypes.byref(o))
    vp = ctypes.c_void_p
    S = (dm.DmuonShape * 1)(dm.DmuonShape(s[0], s[1], dm.DMUON_BF16, dm.DMUON_BF16))
    r = lib.dmuon_muon_step_batched_reduce((vp * 1)(p.data_ptr()), (vp * 2)(g.data_ptr(), None),
                                           (vp * 1)(b.data_ptr()), S, 1, 2, ctypes.byref(o), None, 0, None)
    assert r == -1 and "rank 1" in dm.dmuon_last_error()
    assert lib.dmuon_muon_step_batched_reduce((vp * 1)(p.data_ptr()), (vp * 1)(g.data_ptr()),
                                              (vp * 1)(b.data_ptr()), S, 1, 65, ctypes.byref(o), None, 0,
                                              None) == -1
    torch.cuda.synchronize()
    assert torch.equal(p, p0)
