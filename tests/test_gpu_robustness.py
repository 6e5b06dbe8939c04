"""Checks that stand in for a sanitizer (closed on this pool), on a B200:
* determinism: the same step from the same state gives the same bits (the
  norm reduction is fixed-order, tiles are assigned statically);
* workspace canaries: a step writes nothing outside the caller's scratch,
  checked with guard bytes on both sides of it;
* the optional plan log (DMUON_LOG)."""
import os
import subprocess
import sys

import pytest
import torch

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SHAPES = [((384, 1024), torch.bfloat16), ((1200, 264), torch.bfloat16), ((200, 72), torch.float32),
          ((130, 67), torch.bfloat16), ((4096, 1024), torch.bfloat16), ((1, 9), torch.bfloat16)]
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


def test_two_runs_give_the_same_bits(cuda_lib):
    dm = cuda_lib
    results = []
    for _ in range(2):
        params, grads, bufs = _state(3)
        for _ in range(3):
            dm.dmuon_muon_step_batched(params, grads, bufs, **HP)
        torch.cuda.synchronize()
        results.append([t.clone() for t in params + bufs])
    for a, b in zip(*results):
        assert torch.equal(a, b)


def test_step_writes_nothing_outside_its_workspace(cuda_lib):
    dm = cuda_lib
    params, grads, bufs = _state(5)
    need = dm.dmuon_workspace_bytes(params, HP["ns_steps"], grads)
    guard = 1 << 20
    raw = torch.full((need + 2 * guard,), 0xA5, dtype=torch.uint8, device=DEV)
    ws = raw[guard:guard + need]
    assert ws.data_ptr() % 256 == 0
    for _ in range(2):
        dm.dmuon_muon_step_batched_ex(params, grads, bufs, workspace=ws, **HP)
    torch.cuda.synchronize()
    assert dm.dmuon_device_status() == 0
    assert bool((raw[:guard] == 0xA5).all()) and bool((raw[guard + need:] == 0xA5).all())
    # the caller's tensors themselves: untouched gradients
    _, grads_again, _ = _state(5)
    for g, h in zip(grads, grads_again):
        assert torch.equal(g, h)


def test_plan_log_on_request():
    code = ("import torch, newton_schulz_09_b200 as dm\n"
            "p = [torch.zeros(256, 512, dtype=torch.bfloat16, device='cuda')]\n"
            "g = [torch.ones_like(p[0])]\n"
            "b = [torch.zeros(256, 512, device='cuda')]\n"
            "dm.dmuon_muon_step_batched(p, g, b)\n"
            "torch.cuda.synchronize()\n")
    env = dict(os.environ, DMUON_LOG="1")
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, env=env, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    assert "dmuon: plan on device" in r.stderr and "1 matrices" in r.stderr
    env["DMUON_LOG"] = "0"
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, env=env, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0 and "dmuon: plan" not in r.stderr
