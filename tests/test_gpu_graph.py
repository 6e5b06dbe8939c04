"""CUDA-graph capture of the Muon step (needs a B200).  The first call with a
set of pointers builds the launch plan (host work plus one upload), so it is
made before capture; the captured launches then replay with no host work.
Replays must equal eager steps bit for bit."""
import pytest
import torch

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
SHAPES = [((384, 1024), torch.bfloat16), ((1200, 264), torch.bfloat16), ((200, 72), torch.float32),
          ((4096, 1024), torch.bfloat16)]
HP = dict(lr=0.02, momentum=0.95, nesterov=True, weight_decay=0.01, ns_steps=5)


def _rand(shape, dtype, seed, std=1.0):
    g = torch.Generator(device=DEV)
    g.manual_seed(seed)
    return (torch.randn(shape, generator=g, device=DEV) * std).to(dtype)


def _state(seed):
    params = [_rand(s, d, seed + i, 0.02) for i, (s, d) in enumerate(SHAPES)]
    grads = [_rand(s, d, seed + 10 + i, 1e-3) for i, (s, d) in enumerate(SHAPES)]
    bufs = [_rand(s, torch.float32, seed + 20 + i, 1e-3) for i, (s, d) in enumerate(SHAPES)]
    return params, grads, bufs


def test_captured_step_replays_like_eager(cuda_lib):
    dm = cuda_lib
    params, grads, bufs = _state(1)
    ref_p, ref_b = [p.clone() for p in params], [b.clone() for b in bufs]
    ws = torch.empty(dm.dmuon_workspace_bytes(params, HP["ns_steps"], grads), dtype=torch.uint8, device=DEV)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):                       # eager step: builds the plan
        dm.dmuon_muon_step_batched_ex(params, grads, bufs, workspace=ws, **HP)
    dm.dmuon_muon_step_batched_ex(ref_p, grads, ref_b, **HP)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        dm.dmuon_muon_step_batched_ex(params, grads, bufs, workspace=ws, **HP)
    for step in range(3):
        for i, gr in enumerate(grads):               # new gradients in place between replays
            gr.copy_(_rand(gr.shape, gr.dtype, 100 * step + i, 1e-3))
        g.replay()
        dm.dmuon_muon_step_batched_ex(ref_p, grads, ref_b, **HP)
        torch.cuda.synchronize()
        for i in range(len(SHAPES)):
            assert torch.equal(params[i], ref_p[i]), (step, i)
            assert torch.equal(bufs[i], ref_b[i]), (step, i)
    assert dm.dmuon_device_status() == 0


def test_captured_host_buffer_step(cuda_lib):
    """The host-buffer step forks two copy streams off the caller's stream and
    joins them back, so its copies and kernels are captured as one graph."""
    dm = cuda_lib
    params, _, bufs = _state(2)
    ref_p, ref_b = [p.clone() for p in params], [b.clone() for b in bufs]
    staging = [torch.empty(s, dtype=d, device=DEV) for s, d in SHAPES]
    hg = [torch.empty(s, dtype=d, pin_memory=True) for s, d in SHAPES]
    hw = [torch.empty(s, dtype=d, pin_memory=True) for s, d in SHAPES]
    for i, h in enumerate(hg):
        h.copy_(_rand(h.shape, h.dtype, 50 + i, 1e-3).cpu())
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):                       # eager: plans, scratch and copy streams
        dm.dmuon_muon_step_batched_host(params, staging, bufs, hg, hw, chunks=2, **HP)
    dm.dmuon_muon_step_batched_opts(ref_p, [h.to(DEV) for h in hg], ref_b, **HP)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        dm.dmuon_muon_step_batched_host(params, staging, bufs, hg, hw, chunks=2, **HP)
    for step in range(2):
        for i, h in enumerate(hg):                   # the host fills the pinned buffers
            h.copy_(_rand(h.shape, h.dtype, 200 * step + i, 1e-3).cpu())
        g.replay()
        dm.dmuon_muon_step_batched_opts(ref_p, [h.to(DEV) for h in hg], ref_b, **HP)
        torch.cuda.synchronize()
        for i in range(len(SHAPES)):
            assert torch.equal(params[i], ref_p[i]), (step, i)
            assert torch.equal(bufs[i], ref_b[i]), (step, i)
            assert torch.equal(hw[i], ref_p[i].cpu()), (step, i)


def test_replay_after_eager_calls_with_other_tensors(cuda_lib):
    """Launch plans are cached by shape, and a cached plan's descriptors are
    patched with each call's tensor addresses.  A graph captured on tensors A
    must keep updating A when it is replayed after an eager call on tensors B
    of the same shapes (same workspace, so the same plan); capture also
    refuses shapes that have no plan yet, before anything is enqueued."""
    dm = cuda_lib
    pa, ga, ba = _state(3)
    pb, gb, bb = _state(4)
    ra_p, ra_b = [p.clone() for p in pa], [b.clone() for b in ba]
    rb_p, rb_b = [p.clone() for p in pb], [b.clone() for b in bb]
    ws = torch.empty(dm.dmuon_workspace_bytes(pa, HP["ns_steps"], ga), dtype=torch.uint8, device=DEV)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        dm.dmuon_muon_step_batched_ex(pa, ga, ba, workspace=ws, **HP)     # plan for these shapes
    dm.dmuon_muon_step_batched_ex(ra_p, ga, ra_b, **HP)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        dm.dmuon_muon_step_batched_ex(pa, ga, ba, workspace=ws, **HP)
    with torch.cuda.stream(s):
        dm.dmuon_muon_step_batched_ex(pb, gb, bb, workspace=ws, **HP)     # same plan, tensors B
    dm.dmuon_muon_step_batched_ex(rb_p, gb, rb_b, **HP)
    torch.cuda.synchronize()
    g.replay()                                                             # must update A again
    dm.dmuon_muon_step_batched_ex(ra_p, ga, ra_b, **HP)
    torch.cuda.synchronize()
    with torch.cuda.stream(s):
        dm.dmuon_muon_step_batched_ex(pb, gb, bb, workspace=ws, **HP)     # and B again, eagerly
    dm.dmuon_muon_step_batched_ex(rb_p, gb, rb_b, **HP)
    torch.cuda.synchronize()
    for x, y in zip(pa + ba + pb + bb, ra_p + ra_b + rb_p + rb_b):
        assert torch.equal(x, y)
    # new shapes during a capture: refused, nothing captured
    new_p = [torch.zeros((136, 200), dtype=torch.bfloat16, device=DEV)]
    new_g = [_rand((136, 200), torch.bfloat16, 9, 1e-3)]
    new_b = [torch.zeros((136, 200), dtype=torch.float32, device=DEV)]
    ws2 = torch.empty(dm.dmuon_workspace_bytes(new_p, HP["ns_steps"], new_g), dtype=torch.uint8, device=DEV)
    g2 = torch.cuda.CUDAGraph()
    with pytest.raises(dm.DmuonError) as e:
        with torch.cuda.graph(g2, stream=s):
            dm.dmuon_muon_step_batched_ex(new_p, new_g, new_b, workspace=ws2, **HP)
    assert "capturing" in str(e.value)
    torch.cuda.synchronize()
    assert not new_p[0].any()
    assert dm.dmuon_device_status() == 0
