"""Options of the Muon step against the oracle (needs a B200): custom cubic
coefficients, the per-matrix lr scale 0.2 sqrt(max(rows, cols)), and Muon-only
global-norm gradient clipping before the momentum update."""
import numpy as np
import pytest
import torch

import oracle
from tests.gpu_helpers import TOL_BF16, TOL_F32, check_bf16_weights, check_rel, host

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _rand(shape, dtype, seed, std=1.0):
    g = torch.Generator(device=DEV)
    g.manual_seed(seed)
    return (torch.randn(shape, generator=g, device=DEV) * std).to(dtype)


SHAPES = [(384, 1024), (1200, 264), (256, 256)]


def _inputs(dtype, zero_w, seed=0, gstd=1e-3):
    params = [torch.zeros(s, dtype=dtype, device=DEV) if zero_w else _rand(s, dtype, seed + i, 0.02)
              for i, s in enumerate(SHAPES)]
    grads = [_rand(s, dtype, seed + 10 + i, gstd) for i, s in enumerate(SHAPES)]
    bufs = [_rand(s, torch.float32, seed + 20 + i, gstd) for i, s in enumerate(SHAPES)]
    return params, grads, bufs


def test_default_options_match_the_plain_entry(cuda_lib):
    dm = cuda_lib
    p1, g, b1 = _inputs(torch.bfloat16, False, seed=1)
    p2, b2 = [p.clone() for p in p1], [b.clone() for b in b1]
    dm.dmuon_muon_step_batched(p1, g, b1, lr=0.02, momentum=0.95, nesterov=True,
                               weight_decay=0.01, ns_steps=5)
    dm.dmuon_muon_step_batched_opts(p2, g, b2, lr=0.02, momentum=0.95, nesterov=True,
                                    weight_decay=0.01, ns_steps=5)
    torch.cuda.synchronize()
    for a, b in zip(p1 + b1, p2 + b2):
        assert torch.equal(a, b)


@pytest.mark.parametrize("coeffs", [(1.875, -0.875), (2.0, -1.0)])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32], ids=["bf16", "f32"])
def test_custom_coefficients(cuda_lib, coeffs, dtype):
    dm = cuda_lib
    params, grads, bufs = _inputs(dtype, True, seed=2)
    b0 = [host(b) for b in bufs]
    dm.dmuon_muon_step_batched_opts(params, grads, bufs, lr=0.05, nesterov=True, ns_steps=4,
                                    ns_coefficients=coeffs)
    torch.cuda.synchronize()
    assert dm.dmuon_device_status() == 0
    for i, s in enumerate(SHAPES):
        buf_ref, X, W_ref = oracle.muon_step(np.zeros(s, np.float32), host(grads[i]), b0[i], lr=0.05,
                                             momentum=0.95, nesterov=True, weight_decay=0.0,
                                             ns_steps=4, ns_coeffs=coeffs)
        assert np.array_equal(host(bufs[i]).view(np.uint32), buf_ref.view(np.uint32))
        tol = TOL_BF16 if dtype == torch.bfloat16 else TOL_F32
        check_rel(host(params[i]), W_ref, tol, f"coeffs {coeffs} {s}")


def test_lr_scale_sqrt_max(cuda_lib):
    dm = cuda_lib
    for zero_w in (True, False):
        params, grads, bufs = _inputs(torch.bfloat16, zero_w, seed=3)
        W0 = [host(p) for p in params]
        b0 = [host(b) for b in bufs]
        dm.dmuon_muon_step_batched_opts(params, grads, bufs, lr=0.01, weight_decay=0.05,
                                        lr_scale="sqrt_max")
        torch.cuda.synchronize()
        for i, s in enumerate(SHAPES):
            _, X, W_ref = oracle.muon_step(W0[i], host(grads[i]), b0[i], lr=0.01, momentum=0.95,
                                           nesterov=True, weight_decay=0.05, ns_steps=5,
                                           lr_scale=True)
            if zero_w:
                check_rel(host(params[i]), W_ref, TOL_BF16, f"lr scale {s}")
            else:
                lr_s = 0.01 * oracle.lr_scale_factor(*s)
                check_bf16_weights(host(params[i]), W_ref, X, lr_s, f"lr scale W {s}")


@pytest.mark.parametrize("max_norm", [0.01, 1e6], ids=["clipping", "below-bound"])
def test_gradient_clipping(cuda_lib, max_norm):
    dm = cuda_lib
    # a bf16 group and an fp32 matrix share one global norm
    params, grads, bufs = _inputs(torch.bfloat16, True, seed=4)
    pf = torch.zeros((200, 72), dtype=torch.float32, device=DEV)
    gf = _rand((200, 72), torch.float32, 44, 1e-3)
    bf = _rand((200, 72), torch.float32, 45, 1e-3)
    params, grads, bufs = params + [pf], grads + [gf], bufs + [bf]
    g_host = [host(g) for g in grads]
    b0 = [host(b) for b in bufs]
    norm_out = torch.full((1,), -1.0, dtype=torch.float32, device=DEV)
    dm.dmuon_muon_step_batched_opts(params, grads, bufs, lr=0.02, max_grad_norm=max_norm,
                                    grad_norm_out=norm_out)
    torch.cuda.synchronize()
    assert dm.dmuon_device_status() == 0
    c32, norm = oracle.clip_coefficient(g_host, max_norm)
    assert abs(float(norm_out.item()) - norm) <= 1e-6 * norm
    if max_norm > norm:
        assert c32 == np.float32(1.0)
    for i in range(len(params)):
        buf_ref, X, W_ref = oracle.muon_step(np.zeros(g_host[i].shape, np.float32), g_host[i], b0[i],
                                             lr=0.02, momentum=0.95, nesterov=True,
                                             weight_decay=0.0, ns_steps=5, grad_scale=c32)
        assert np.array_equal(host(bufs[i]).view(np.uint32), buf_ref.view(np.uint32)), i
        tol = TOL_BF16 if params[i].dtype == torch.bfloat16 else TOL_F32
        check_rel(host(params[i]), W_ref, tol, f"clip {max_norm} [{i}]")
    # gradients are read only
    for g, gh in zip(grads, g_host):
        assert np.array_equal(host(g), gh)


QUINTIC = [(3.4445, -4.7750, 2.0315), (15.0 / 8.0, -10.0 / 8.0, 3.0 / 8.0)]


@pytest.mark.parametrize("coeffs", QUINTIC, ids=["jordan", "textbook"])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32], ids=["bf16", "f32"])
@pytest.mark.parametrize("steps", [1, 5])
def test_quintic_coefficients(cuda_lib, coeffs, dtype, steps):
    """X <- a X + b A X + c A^2 X (A = X X^T): the SYRK, the symmetric square
    P = b A + c A A and the GEMM X <- a X + P X, against the oracle's quintic
    step; tall, square and multi-band wide shapes with ragged sizes."""
    dm = cuda_lib
    shapes = [(384, 1024), (1200, 264), (256, 256), (520, 600)]
    params = [torch.zeros(s, dtype=dtype, device=DEV) for s in shapes]
    grads = [_rand(s, dtype, 60 + i, 1e-3) for i, s in enumerate(shapes)]
    bufs = [_rand(s, torch.float32, 70 + i, 1e-3) for i, s in enumerate(shapes)]
    b0 = [host(b) for b in bufs]
    dm.dmuon_muon_step_batched_opts(params, grads, bufs, lr=0.05, nesterov=True, ns_steps=steps,
                                    ns_coefficients=coeffs)
    torch.cuda.synchronize()
    assert dm.dmuon_device_status() == 0
    for i, s in enumerate(shapes):
        buf_ref, X, W_ref = oracle.muon_step(np.zeros(s, np.float32), host(grads[i]), b0[i], lr=0.05,
                                             momentum=0.95, nesterov=True, weight_decay=0.0,
                                             ns_steps=steps, ns_coeffs=coeffs)
        assert np.array_equal(host(bufs[i]).view(np.uint32), buf_ref.view(np.uint32))
        tol = TOL_BF16 if dtype == torch.bfloat16 else TOL_F32
        check_rel(host(params[i]), W_ref, tol, f"quintic {coeffs} {s} k={steps}")


def test_quintic_caller_workspace_size(cuda_lib):
    """The quintic step needs one more m x m matrix of scratch: the size query
    with the options says so, and a workspace of exactly that size works."""
    dm = cuda_lib
    import ctypes
    shapes = [(300, 700), (900, 130)]
    S = (dm.DmuonShape * 2)(*[dm.DmuonShape(r, c, dm.DMUON_BF16, dm.DMUON_BF16) for r, c in shapes])
    lib = dm.load_library()
    o = dm.DmuonStepOptions()
    lib.dmuon_step_options_default(ctypes.byref(o))
    cubic = lib.dmuon_workspace_bytes_opts(S, 2, ctypes.byref(o))
    assert cubic == lib.dmuon_workspace_bytes(S, 2, 5)
    o.ns_a, o.ns_b, o.ns_c = QUINTIC[0]
    need = lib.dmuon_workspace_bytes_opts(S, 2, ctypes.byref(o))
    assert need >= cubic + 2 * (300 * 304 + 130 * 136)
    params = [torch.zeros(s, dtype=torch.bfloat16, device=DEV) for s in shapes]
    grads = [_rand(s, torch.bfloat16, 80 + i, 1e-3) for i, s in enumerate(shapes)]
    bufs = [torch.zeros(s, dtype=torch.float32, device=DEV) for s in shapes]
    p2, b2 = [p.clone() for p in params], [b.clone() for b in bufs]
    ws = torch.empty(need, dtype=torch.uint8, device=DEV)
    dm.dmuon_muon_step_batched_opts(params, grads, bufs, ns_coefficients=QUINTIC[0], workspace=ws)
    dm.dmuon_muon_step_batched_opts(p2, grads, b2, ns_coefficients=QUINTIC[0])
    torch.cuda.synchronize()
    for a, b in zip(params + bufs, p2 + b2):
        assert torch.equal(a, b)
    with pytest.raises(dm.DmuonError):
        dm.dmuon_muon_step_batched_opts(params, grads, bufs, ns_coefficients=QUINTIC[0],
                                        workspace=ws[:cubic])


@pytest.mark.slow
def test_quintic_on_the_large_tile_syrk(cuda_lib):
    """A 4096 x 4096 matrix runs its SYRK with 256 x 256 tiles (136 tiles in one
    wave against 272 small ones in two) and its GEMM on CTA pairs; in the
    quintic step the SQUARE stage reads A's upper triangle, the k-blocks left
    of each operand's diagonal 256-block transposed.  Against the oracle's
    quintic step."""
    dm = cuda_lib
    s = (4096, 4096)
    p = torch.zeros(s, dtype=torch.bfloat16, device=DEV)
    g = _rand(s, torch.bfloat16, 90, 1e-3)
    b = torch.zeros(s, dtype=torch.float32, device=DEV)
    dm.dmuon_muon_step_batched_opts([p], [g], [b], lr=0.05, nesterov=True, ns_steps=3,
                                    ns_coefficients=QUINTIC[0])
    torch.cuda.synchronize()
    assert dm.dmuon_device_status() == 0
    buf_ref, X, W_ref = oracle.muon_step(np.zeros(s, np.float32), host(g), np.zeros(s, np.float32), lr=0.05,
                                         momentum=0.95, nesterov=True, weight_decay=0.0, ns_steps=3,
                                         ns_coeffs=QUINTIC[0])
    assert np.array_equal(host(b).view(np.uint32), buf_ref.view(np.uint32))
    check_rel(host(p), W_ref, TOL_BF16, "quintic 4096^2 (256 x 256 SYRK tiles)")
