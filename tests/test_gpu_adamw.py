"""AdamW of the non-orthogonalised parameters against the oracle (needs a B200):
several steps over tensors of mixed sizes and dtypes in one call; moments
bit-exact, parameters within one storage ulp of the fp64 result."""
import numpy as np
import pytest
import torch

import oracle
from tests.gpu_helpers import bf16_ulp, host

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _rand(shape, dtype, seed, std=1.0):
    g = torch.Generator(device=DEV)
    g.manual_seed(seed)
    return (torch.randn(shape, generator=g, device=DEV) * std).to(dtype)


CASES = [  # shape, param dtype, grad dtype
    ((4096,), torch.bfloat16, torch.bfloat16),      # norm weight
    ((128, 1000), torch.bfloat16, torch.bfloat16),  # small head, ragged
    ((333,), torch.float32, torch.float32),         # ragged fp32 bias
    ((2049,), torch.float32, torch.bfloat16),       # fp32 master with bf16 grad
    ((3_000_001,), torch.bfloat16, torch.bfloat16), # large, many work items
    ((7,), torch.bfloat16, torch.bfloat16),         # tiny
]


def _check_param(got, want, prev, lr, dtype, what, ulps):
    """The kernel evaluates the update in fp32: its error is a few fp32
    roundings of the operands (|p| and the step, which is at most ~lr), which
    matters where the update cancels the weight.  bf16 storage adds `ulps`
    bf16 ulps of the result."""
    got64 = got.astype(np.float64)
    err = np.abs(got64 - want)
    tol = ulps * 2.0 ** -23 * (np.abs(prev) + np.abs(want) + 4.0 * lr)
    if dtype == torch.bfloat16:
        tol = tol + ulps * np.maximum(bf16_ulp(want), bf16_ulp(got64)) * (1 + 1e-6)
    bad = err > tol
    if bad.any():
        i = int(np.argmax(err / tol))
        raise AssertionError(f"{what}: {int(bad.sum())} elements off; worst at {i}: got {got64.flat[i]!r} "
                             f"want {want.flat[i]!r} prev {np.asarray(prev).flat[i]!r} tol {tol.flat[i]:.3e}")


def _stored(x64, dtype):
    """The oracle's own copy of the parameter in its storage dtype."""
    return torch.from_numpy(np.asarray(x64)).to(dtype).to(torch.float64).numpy()


def test_adamw_three_steps(cuda_lib):
    dm = cuda_lib
    params = [_rand(s, pd, 10 + i, 0.02) for i, (s, pd, gd) in enumerate(CASES)]
    ms = [torch.zeros(s, dtype=torch.float32, device=DEV) for s, _, _ in CASES]
    vs = [torch.zeros(s, dtype=torch.float32, device=DEV) for s, _, _ in CASES]
    ref = [(host(p).astype(np.float64), np.zeros(p.shape, np.float32), np.zeros(p.shape, np.float32))
           for p in params]
    hp = dict(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.01)
    for step in (1, 2, 3):
        grads = [_rand(s, gd, 100 * step + i, 1e-3 * (i + 1)) for i, (s, pd, gd) in enumerate(CASES)]
        if step == 2:
            grads[2] = None                       # skipped this step
        dm.dmuon_adamw_step_batched(params, grads, ms, vs, lr=hp["lr"], betas=(hp["beta1"], hp["beta2"]),
                                    eps=hp["eps"], weight_decay=hp["weight_decay"], step=step)
        torch.cuda.synchronize()
        for i, (s, pd, gd) in enumerate(CASES):
            p_ref, m_ref, v_ref = ref[i]
            if grads[i] is not None:
                # the oracle keeps its own parameter, rounded to the storage dtype
                m_ref, v_ref, p_new = oracle.adamw_step(p_ref, host(grads[i]), m_ref, v_ref, step=step, **hp)
                _check_param(host(params[i]), p_new, p_ref, hp["lr"], pd, f"step {step} tensor {i}", ulps=step)
                ref[i] = (_stored(p_new, pd), m_ref, v_ref)
            assert np.array_equal(host(ms[i]).view(np.uint32), m_ref.view(np.uint32)), (step, i)
            assert np.array_equal(host(vs[i]).view(np.uint32), v_ref.view(np.uint32)), (step, i)


def test_adamw_rejects_bad_arguments(cuda_lib):
    dm = cuda_lib
    p = _rand((16,), torch.float32, 1)
    g = _rand((16,), torch.float32, 2)
    m = torch.zeros(16, device=DEV)
    v = torch.zeros(16, device=DEV)
    for kw in (dict(step=0), dict(betas=(1.0, 0.999)), dict(eps=0.0)):
        with pytest.raises(dm.DmuonError):
            dm.dmuon_adamw_step_batched([p], [g], [m], [v], **kw)
    with pytest.raises(ValueError):
        dm.dmuon_adamw_step_batched([p], [g], [m.to(torch.bfloat16)], [v])
