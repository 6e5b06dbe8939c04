"""The host-buffer Muon step (needs a B200): gradients uploaded from pinned
host memory and weights downloaded to it, overlapped with the update in
groups.  The device results must equal the device-only entry point bit for
bit (same kernels per matrix), the downloaded weights must equal the device
weights, and a small case is checked against the oracle."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from tests.gpu_helpers import TOL_BF16, TOL_F32, check_bf16_weights, check_rel, host

pytestmark = pytest.mark.gpu

DEV = "cuda:0"

# bf16 and fp32 matrices, tall (transposed) and wide, ragged sizes
SHAPES = [((384, 1024), torch.bfloat16), ((1200, 264), torch.bfloat16), ((256, 256), torch.bfloat16),
          ((200, 72), torch.float32), ((520, 1032), torch.bfloat16), ((64, 4096), torch.bfloat16)]


def _rand(shape, dtype, seed, std=1.0):
    g = torch.Generator(device=DEV)
    g.manual_seed(seed)
    return (torch.randn(shape, generator=g, device=DEV) * std).to(dtype)


def _state(seed):
    params = [_rand(s, d, seed + i, 0.02) for i, (s, d) in enumerate(SHAPES)]
    bufs = [_rand(s, torch.float32, seed + 20 + i, 1e-3) for i, (s, d) in enumerate(SHAPES)]
    return params, bufs


def _host_grads(seed):
    out = []
    for i, (s, d) in enumerate(SHAPES):
        h = torch.empty(s, dtype=d, pin_memory=True)
        h.copy_(_rand(s, d, seed + 40 + i, 1e-3).cpu())
        out.append(h)
    return out


HP = dict(lr=0.02, momentum=0.95, nesterov=True, weight_decay=0.01, ns_steps=5)


@pytest.mark.parametrize("chunks", [1, 2, 0, len(SHAPES)], ids=["one", "two", "auto", "per-matrix"])
def test_matches_device_entry_bitwise(cuda_lib, chunks):
    dm = cuda_lib
    params, bufs = _state(1)
    ref_p, ref_b = [p.clone() for p in params], [b.clone() for b in bufs]
    staging = [torch.empty(s, dtype=d, device=DEV) for s, d in SHAPES]
    host_out = [torch.empty(s, dtype=d, pin_memory=True) for s, d in SHAPES]
    for step in range(2):                      # two steps: state carries over
        hg = _host_grads(100 * step)
        dm.dmuon_muon_step_batched_host(params, staging, bufs, hg, host_out, chunks=chunks, **HP)
        dev_g = [h.to(DEV) for h in hg]
        dm.dmuon_muon_step_batched_opts(ref_p, dev_g, ref_b, **HP)
        torch.cuda.synchronize()
        assert dm.dmuon_device_status() == 0
        for i in range(len(SHAPES)):
            assert torch.equal(params[i], ref_p[i]), (step, i)
            assert torch.equal(bufs[i], ref_b[i]), (step, i)
            assert torch.equal(host_out[i], params[i].cpu()), (step, i)
            assert torch.equal(staging[i].cpu(), hg[i]), (step, i)


def test_against_oracle(cuda_lib):
    dm = cuda_lib
    params, bufs = _state(7)
    W0 = [host(p) for p in params]
    b0 = [host(b) for b in bufs]
    hg = _host_grads(7)
    staging = [torch.empty(s, dtype=d, device=DEV) for s, d in SHAPES]
    host_out = [torch.empty(s, dtype=d, pin_memory=True) for s, d in SHAPES]
    dm.dmuon_muon_step_batched_host(params, staging, bufs, hg, host_out, chunks=3, **HP)
    torch.cuda.synchronize()
    for i, (s, d) in enumerate(SHAPES):
        buf_ref, X, W_ref = oracle.muon_step(W0[i], host(hg[i]), b0[i], **HP)
        assert np.array_equal(host(bufs[i]).view(np.uint32), buf_ref.view(np.uint32)), i
        if d == torch.bfloat16:
            check_bf16_weights(host(host_out[i]), W_ref, X, HP["lr"], f"host W {s}")
        else:
            check_rel(host(host_out[i]) - W0[i], W_ref - W0[i], TOL_F32, f"host dW {s}")


def test_skips_and_optional_download(cuda_lib):
    dm = cuda_lib
    params, bufs = _state(3)
    p0, b0 = [p.clone() for p in params], [b.clone() for b in bufs]
    staging = [torch.empty(s, dtype=d, device=DEV) for s, d in SHAPES]
    hg = _host_grads(3)
    hg[1] = None                                   # no gradient: matrix 1 untouched
    host_out = [torch.full(s, 7.0, dtype=d).pin_memory() for s, d in SHAPES]
    host_out[2] = None                             # updated on the device, not downloaded
    dm.dmuon_muon_step_batched_host(params, staging, bufs, hg, host_out, chunks=2, **HP)
    torch.cuda.synchronize()
    assert torch.equal(params[1], p0[1]) and torch.equal(bufs[1], b0[1])
    assert bool((host_out[1] == 7.0).all())       # skipped matrices are not downloaded
    assert not torch.equal(bufs[2], b0[2])
    for i in (0, 3, 4, 5):
        assert torch.equal(host_out[i], params[i].cpu())


def test_rejects_pageable_host_memory(cuda_lib):
    dm = cuda_lib
    params, bufs = _state(5)
    staging = [torch.empty(s, dtype=d, device=DEV) for s, d in SHAPES]
    pageable = [torch.zeros(s, dtype=d) for s, d in SHAPES]
    with pytest.raises(ValueError):
        dm.dmuon_muon_step_batched_host(params, staging, bufs, pageable, None, **HP)
    # the C ABI checks on its own: a pageable buffer passed straight through
    lib = dm.load_library()
    o = dm.DmuonStepOptions()
    lib.dmuon_step_options_default(ctypes.byref(o))
    page = np.zeros(16, np.float32)
    vp = ctypes.c_void_p
    arr = lambda *v: (vp * len(v))(*v)
    S = (dm.DmuonShape * 1)(dm.DmuonShape(4, 4, dm.DMUON_F32, dm.DMUON_F32))
    p = torch.zeros((4, 4), device=DEV)
    g = torch.zeros((4, 4), device=DEV)
    b = torch.zeros((4, 4), device=DEV)
    r = lib.dmuon_muon_step_batched_host(arr(p.data_ptr()), arr(g.data_ptr()), arr(b.data_ptr()),
                                         arr(page.ctypes.data), arr(None), S, 1, ctypes.byref(o), 0,
                                         None, 0, None)
    assert r == -2 and "page-locked" in dm.dmuon_last_error()
    assert torch.equal(b, torch.zeros_like(b))
