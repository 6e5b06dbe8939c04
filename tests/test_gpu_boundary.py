"""The entry points only enqueue (needs a B200).

Launch plans depend on shapes, not on tensor addresses: new addresses are
patched into a cached plan in stream order, so a training loop whose
gradients move every step builds no new plan.  Plan builds, arena growth and
plan eviction never wait for the device: a call returns while the stream is
still busy with earlier work.  Host memory is refused before anything is
enqueued.
"""
import ctypes

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
SHAPES = [(384, 1024, torch.bfloat16), (1200, 264, torch.bfloat16), (256, 256, torch.float32),
          (96, 700, torch.bfloat16), (520, 136, torch.float32), (1024, 1024, torch.bfloat16)]


def _rand(shape, dtype, seed, std):
    g = torch.Generator(device=DEV)
    g.manual_seed(seed)
    return (torch.randn(shape, generator=g, device=DEV) * std).to(dtype)


def _state(seed):
    params = [_rand((r, c), dt, seed + i, 0.02) for i, (r, c, dt) in enumerate(SHAPES)]
    bufs = [torch.zeros((r, c), dtype=torch.float32, device=DEV) for r, c, _ in SHAPES]
    return params, bufs


def _grads(step):
    return [_rand((r, c), dt, 1000 * step + i, 1e-3) for i, (r, c, dt) in enumerate(SHAPES)]


def test_new_addresses_every_step_build_no_plan(cuda_lib):
    dm = cuda_lib
    steps = 100
    # reference: the same tensors (addresses) every step
    p_ref, b_ref = _state(1)
    g_fixed = _grads(0)
    for s in range(steps):
        for g, src in zip(g_fixed, _grads(s)):
            g.copy_(src)
        dm.dmuon_muon_step_batched(p_ref, g_fixed, b_ref, lr=0.02, weight_decay=0.01)
    torch.cuda.synchronize()
    builds0 = dm.dmuon_plan_builds()
    # moving: every step new gradient tensors (all kept alive, so the
    # allocator cannot hand back the same blocks), and every tenth step the
    # parameters and buffers move too
    p, b = _state(1)
    keep = []
    addrs = set()
    for s in range(steps):
        grads = _grads(s)
        keep.append(grads)
        if s % 10 == 5:
            p = [t.clone() for t in p]
            b = [t.clone() for t in b]
        addrs.add(tuple(g.data_ptr() for g in grads))
        dm.dmuon_muon_step_batched(p, grads, b, lr=0.02, weight_decay=0.01)
    torch.cuda.synchronize()
    assert dm.dmuon_device_status() == 0
    assert len(addrs) == steps                              # the addresses did move
    assert dm.dmuon_plan_builds() == builds0, "a step with new addresses built a plan"
    for a, r in zip(p + b, p_ref + b_ref):
        assert torch.equal(a, r)


def test_calls_return_while_the_stream_is_busy(cuda_lib):
    """Plan builds (new shapes), arena growth and plan eviction (more than 64
    plans) enqueue without waiting: the calls return before a long kernel
    queued ahead of them has finished."""
    dm = cuda_lib
    torch.cuda.synchronize()
    st = torch.cuda.current_stream()
    torch.cuda._sleep(int(3e9))          # about two seconds of GPU clock cycles
    n_shapes = 70                         # more than the plan cache holds
    results = []
    for k in range(n_shapes):
        r, c = 64 + 8 * k, 128 + 16 * (k % 9)
        p = torch.zeros((r, c), dtype=torch.bfloat16, device=DEV)
        g = _rand((r, c), torch.bfloat16, 500 + k, 1e-3)
        b = torch.zeros((r, c), dtype=torch.float32, device=DEV)
        dm.dmuon_muon_step_batched([p], [g], [b], lr=0.02, ns_steps=2)
        results.append((p, g, b))
    # a much larger call grows the arena
    big = [torch.zeros((2048, 4096), dtype=torch.bfloat16, device=DEV)]
    bg = [_rand((2048, 4096), torch.bfloat16, 900, 1e-3)]
    bb = [torch.zeros((2048, 4096), dtype=torch.float32, device=DEV)]
    dm.dmuon_muon_step_batched(big, bg, bb, lr=0.02)
    busy = not st.query()
    torch.cuda.synchronize()
    assert busy, "a call waited for the device"
    assert dm.dmuon_device_status() == 0
    # the results equal a second, unhurried run of the same calls
    for k, (p, g, b) in enumerate(results):
        p2, b2 = torch.zeros_like(p), torch.zeros_like(b)
        dm.dmuon_muon_step_batched([p2], [g], [b2], lr=0.02, ns_steps=2)
        torch.cuda.synchronize()
        assert torch.equal(p, p2) and torch.equal(b, b2), k


def test_plan_used_on_two_streams_with_one_workspace(cuda_lib):
    """A caller workspace shared by two streams: the second stream's call is
    ordered after the first's use of the plan (no race on the scratch)."""
    dm = cuda_lib
    shapes = [(512, 1024), (1024, 384)]
    ws = torch.empty(dm.dmuon_workspace_bytes([torch.empty(s) for s in shapes], 5), dtype=torch.uint8,
                     device=DEV)

    def make(seed):
        p = [torch.zeros(s, dtype=torch.bfloat16, device=DEV) for s in shapes]
        g = [_rand(s, torch.bfloat16, seed + i, 1e-3) for i, s in enumerate(shapes)]
        b = [torch.zeros(s, dtype=torch.float32, device=DEV) for s in shapes]
        return p, g, b

    a, bset = make(10), make(20)
    ra, rb = make(10), make(20)
    torch.cuda.synchronize()
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    with torch.cuda.stream(s1):
        torch.cuda._sleep(int(1e9))
        dm.dmuon_muon_step_batched_ex(*a, workspace=ws)
    with torch.cuda.stream(s2):
        dm.dmuon_muon_step_batched_ex(*bset, workspace=ws)
    torch.cuda.synchronize()
    dm.dmuon_muon_step_batched(*ra)
    dm.dmuon_muon_step_batched(*rb)
    torch.cuda.synchronize()
    for x, y in zip(a[0] + a[2] + bset[0] + bset[2], ra[0] + ra[2] + rb[0] + rb[2]):
        assert torch.equal(x, y)


def test_host_memory_is_refused_before_anything_is_enqueued(cuda_lib):
    dm = cuda_lib
    dev_t = torch.zeros(64, device=DEV)
    pinned = torch.zeros(64, pin_memory=True)
    pageable = np.zeros(64, dtype=np.float32)
    assert dm.dmuon_debug_check_pointer(dev_t.data_ptr()) == 0
    assert dm.dmuon_debug_check_pointer(pinned.data_ptr()) == -1
    assert dm.dmuon_debug_check_pointer(pageable.ctypes.data) == -1
    assert dm.dmuon_debug_check_pointer(0) == -1
    # a page-locked host gradient through the entry point: refused, nothing runs
    p = torch.zeros((128, 256), dtype=torch.bfloat16, device=DEV)
    b = torch.zeros((128, 256), dtype=torch.float32, device=DEV)
    hg = torch.ones((128, 256), dtype=torch.bfloat16, pin_memory=True)
    lib = dm.load_library()
    n0 = dm.dmuon_launch_count()
    P = (ctypes.c_void_p * 1)(p.data_ptr())
    G = (ctypes.c_void_p * 1)(hg.data_ptr())
    B = (ctypes.c_void_p * 1)(b.data_ptr())
    S = (dm.DmuonShape * 1)(dm.DmuonShape(128, 256, dm.DMUON_BF16, dm.DMUON_BF16))
    r = lib.dmuon_muon_step_batched(P, G, B, S, 1, 0.02, 0.95, 1, 0.0, 5, None)
    assert r == -1 and "not device memory" in dm.dmuon_last_error()
    # the clip and AdamW entry points check their tensors too
    D = (dm.DmuonGradDesc * 1)(dm.DmuonGradDesc(hg.numel(), dm.DMUON_BF16, 0))
    M = (ctypes.c_float * 1)(1.0)
    r = lib.dmuon_clip_grad_norm_buckets(G, D, 1, M, 1, None, None, None, 0, None)
    assert r == -1 and "not device memory" in dm.dmuon_last_error()
    m = torch.zeros(hg.numel(), dtype=torch.float32, device=DEV)
    v = torch.zeros(hg.numel(), dtype=torch.float32, device=DEV)
    TD = (dm.DmuonTensorDesc * 1)(dm.DmuonTensorDesc(hg.numel(), dm.DMUON_BF16, dm.DMUON_BF16))
    pp = ctypes.POINTER(ctypes.c_void_p)
    r = lib.dmuon_adamw_step_batched(ctypes.cast(P, pp), ctypes.cast(G, pp),
                                     ctypes.cast((ctypes.c_void_p * 1)(m.data_ptr()), pp),
                                     ctypes.cast((ctypes.c_void_p * 1)(v.data_ptr()), pp),
                                     TD, 1, 1e-3, 0.9, 0.999, 1e-8, 0.0, 1, None)
    assert r == -1 and "not device memory" in dm.dmuon_last_error()
    assert dm.dmuon_launch_count() == n0
    torch.cuda.synchronize()
    assert not p.any() and not b.any()
