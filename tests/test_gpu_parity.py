"""CUDA path against the fp64 oracle on the same seeded inputs (needs a B200).

Sizes span several 128 x 256 tiles with ragged tails, both orientations
(rows > cols runs on the transposed view), and the degenerate cases: one
element, one row, zero input, NaN input, zero steps, one step.
"""
import numpy as np
import pytest
import torch

import oracle
from newton_schulz_09_b200 import synthetic
from tests.gpu_helpers import (TOL_BF16, TOL_F32, check_bf16_weights, check_rel, host,
                               oracle_step, tol_for)

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _rand(shape, dtype, seed, std=1.0):
    g = torch.Generator(device=DEV)
    g.manual_seed(seed)
    return (torch.randn(shape, generator=g, device=DEV) * std).to(dtype)


ORTHO_SHAPES = [
    (128, 256), (256, 512), (512, 256), (384, 384), (200, 328), (328, 200), (1, 1), (1, 9),
    (9, 1), (3, 5), (100, 1000), (1000, 100), (64, 2048), (130, 390), (520, 1040), (257, 513),
    # long side a multiple of 64 but not of 256: the last column tile of the GEMM's
    # B operand is partly past the matrix (3-D loads fill it with zeros)
    (320, 640), (448, 192), (704, 2112),
]


@pytest.mark.parametrize("shape", ORTHO_SHAPES, ids=lambda s: f"{s[0]}x{s[1]}")
@pytest.mark.parametrize("steps", [0, 1, 5])
def test_orthogonalize_bf16(cuda_lib, shape, steps):
    dm = cuda_lib
    G = _rand(shape, torch.bfloat16, seed=shape[0] * 7919 + shape[1])
    want = oracle.newton_schulz(host(G), steps)
    X = G.clone()
    dm.dmuon_ns_orthogonalize(X, steps)
    torch.cuda.synchronize()
    assert dm.dmuon_device_status() == 0
    check_rel(host(X), want, TOL_BF16, f"NS bf16 {shape} k={steps}")


@pytest.mark.parametrize("shape", [(256, 512), (512, 256), (200, 328), (1, 7), (130, 390), (64, 1024)],
                         ids=lambda s: f"{s[0]}x{s[1]}")
@pytest.mark.parametrize("steps", [0, 1, 5])
def test_orthogonalize_f32(cuda_lib, shape, steps):
    dm = cuda_lib
    G = _rand(shape, torch.float32, seed=shape[0] * 31 + shape[1])
    want = oracle.newton_schulz(host(G), steps)
    X = G.clone()
    dm.dmuon_ns_orthogonalize_ex(X, steps)
    torch.cuda.synchronize()
    assert dm.dmuon_device_status() == 0
    check_rel(host(X), want, TOL_F32, f"NS f32 {shape} k={steps}")


def test_orthogonalize_is_deterministic(cuda_lib):
    dm = cuda_lib
    G = _rand((520, 1040), torch.bfloat16, seed=5)
    a, b = G.clone(), G.clone()
    dm.dmuon_ns_orthogonalize(a, 5)
    dm.dmuon_ns_orthogonalize(b, 5)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


def test_zero_input_gives_zero(cuda_lib):
    dm = cuda_lib
    X = torch.zeros((300, 700), dtype=torch.bfloat16, device=DEV)
    dm.dmuon_ns_orthogonalize(X, 5)
    torch.cuda.synchronize()
    assert torch.count_nonzero(X).item() == 0


def test_nan_input_propagates_without_hanging(cuda_lib):
    dm = cuda_lib
    X = _rand((256, 512), torch.bfloat16, seed=9)
    X[3, 7] = float("nan")
    dm.dmuon_ns_orthogonalize(X, 5)
    torch.cuda.synchronize()
    assert dm.dmuon_device_status() == 0
    assert torch.isnan(X.float()).any()


# ------------------------------------------------------------------ Muon step
def _run_step(dm, wl, t, lr=None):
    dm.dmuon_muon_step_batched(t.params, t.grads, t.bufs, lr=wl.lr if lr is None else lr,
                               momentum=wl.momentum, nesterov=wl.nesterov,
                               weight_decay=wl.weight_decay, ns_steps=wl.ns_steps)


def test_fp32_256x512_step(cuda_lib):
    """One fp32 256x512 matrix, N(0,1) gradient, zero buffer, Nesterov, 5 steps."""
    dm = cuda_lib
    wl = synthetic.workload("fp32_256x512")
    t = synthetic.make_tensors(wl, device=DEV)
    W0, g0, b0 = t.params[0].clone(), t.grads[0].clone(), t.bufs[0].clone()
    _run_step(dm, wl, t)
    torch.cuda.synchronize()
    assert dm.dmuon_device_status() == 0
    buf_ref, X_ref, W_ref = oracle_step(W0, g0, b0, lr=wl.lr, momentum=wl.momentum,
                                        nesterov=wl.nesterov, weight_decay=wl.weight_decay,
                                        ns_steps=wl.ns_steps)
    assert np.array_equal(host(t.bufs[0]).view(np.uint32), buf_ref.view(np.uint32))
    dW = host(t.params[0]).astype(np.float64) - host(W0)
    check_rel(dW, W_ref - host(W0), TOL_F32, "fp32 update W' - W")


def test_tinymlp_with_momentum_history(cuda_lib):
    """TinyMLP shapes; three prior momentum steps (lr = 0, so W is untouched
    and only the buffers evolve), then the measured step."""
    dm = cuda_lib
    wl = synthetic.workload("tinymlp")
    t = synthetic.make_tensors(wl, device=DEV)
    W0 = [p.clone() for p in t.params]
    bufs_ref = [host(b) for b in t.bufs]
    for s in range(wl.prior_steps):
        step = synthetic.Tensors(t.params, t.prior_grads[s], t.bufs, [])
        _run_step(dm, wl, step, lr=0.0)
        torch.cuda.synchronize()
        for i in range(len(t.params)):
            bufs_ref[i] = oracle.momentum_update(bufs_ref[i], host(t.prior_grads[s][i]), wl.momentum)
            assert np.array_equal(host(t.bufs[i]).view(np.uint32), bufs_ref[i].view(np.uint32)), (s, i)
            assert torch.equal(t.params[i], W0[i])
    bufs_before = [b.copy() for b in bufs_ref]
    _run_step(dm, wl, t)
    torch.cuda.synchronize()
    assert dm.dmuon_device_status() == 0
    for i in range(len(t.params)):
        buf_ref, X_ref, W_ref = oracle.muon_step(host(W0[i]), host(t.grads[i]), bufs_before[i],
                                                 lr=wl.lr, momentum=wl.momentum,
                                                 nesterov=wl.nesterov,
                                                 weight_decay=wl.weight_decay,
                                                 ns_steps=wl.ns_steps)
        assert np.array_equal(host(t.bufs[i]).view(np.uint32), buf_ref.view(np.uint32)), i
        check_bf16_weights(host(t.params[i]), W_ref, X_ref, wl.lr, f"tinymlp W[{i}]")


@pytest.mark.parametrize("shape", [(2048, 512), (512, 2048), (300, 1000), (1000, 300), (640, 640)],
                         ids=lambda s: f"{s[0]}x{s[1]}")
def test_update_reveals_x_through_zero_weights(cuda_lib, shape):
    """With W = 0 the step writes bf16(-lr X): the orthogonalised matrix of the
    Muon path itself, checked at the bf16 tolerance."""
    dm = cuda_lib
    g = _rand(shape, torch.bfloat16, seed=shape[0] + 3 * shape[1], std=1e-3)
    buf = _rand(shape, torch.float32, seed=shape[1], std=2e-3)
    W = torch.zeros(shape, dtype=torch.bfloat16, device=DEV)
    bufs_h = host(buf)
    dm.dmuon_muon_step_batched([W], [g], [buf], lr=0.02, momentum=0.95, nesterov=True,
                               weight_decay=0.1, ns_steps=5)
    torch.cuda.synchronize()
    buf_ref, X_ref, W_ref = oracle.muon_step(np.zeros(shape, np.float32), host(g), bufs_h, lr=0.02,
                                             momentum=0.95, nesterov=True, weight_decay=0.1,
                                             ns_steps=5)
    assert np.array_equal(host(buf).view(np.uint32), buf_ref.view(np.uint32))
    check_rel(host(W), W_ref, TOL_BF16, f"-lr X {shape}")


def test_mixed_batch_with_skips_and_both_dtypes(cuda_lib):
    """bf16 and fp32 parameters in one call, a fp32 gradient on a bf16 weight,
    a matrix without gradient (left untouched), ragged and tall shapes."""
    dm = cuda_lib
    shapes = [(256, 520), (600, 136), (64, 64), (333, 77), (128, 4096)]
    dts = [torch.bfloat16, torch.bfloat16, torch.float32, torch.float32, torch.bfloat16]
    gdts = [torch.bfloat16, torch.float32, torch.float32, torch.float32, torch.bfloat16]
    params, grads, bufs = [], [], []
    for i, (s, dt, gdt) in enumerate(zip(shapes, dts, gdts)):
        params.append(_rand(s, dt, 100 + i, 0.02))
        grads.append(_rand(s, gdt, 200 + i, 1e-2))
        bufs.append(_rand(s, torch.float32, 300 + i, 1e-2))
    grads[3] = None
    P0 = [p.clone() for p in params]
    B0 = [b.clone() for b in bufs]
    dm.dmuon_muon_step_batched(params, grads, bufs, lr=0.05, momentum=0.9, nesterov=False,
                               weight_decay=0.01, ns_steps=4)
    torch.cuda.synchronize()
    assert dm.dmuon_device_status() == 0
    for i in range(len(shapes)):
        if grads[i] is None:
            assert torch.equal(params[i], P0[i]) and torch.equal(bufs[i], B0[i])
            continue
        buf_ref, X_ref, W_ref = oracle.muon_step(host(P0[i]), host(grads[i]), host(B0[i]),
                                                 lr=0.05, momentum=0.9, nesterov=False,
                                                 weight_decay=0.01, ns_steps=4)
        assert np.array_equal(host(bufs[i]).view(np.uint32), buf_ref.view(np.uint32)), i
        if dts[i] == torch.bfloat16:
            check_bf16_weights(host(params[i]), W_ref, X_ref, 0.05, f"mixed W[{i}]")
        else:
            check_rel(host(params[i]).astype(np.float64) - host(P0[i]), W_ref - host(P0[i]), TOL_F32,
                      f"mixed fp32 dW[{i}]")


def test_ex_entry_with_torch_workspace_matches_arena(cuda_lib):
    dm = cuda_lib
    shapes = [(384, 1024), (1024, 384)]
    ps = [_rand(s, torch.bfloat16, 7 + i, 0.02) for i, s in enumerate(shapes)]
    gs = [_rand(s, torch.bfloat16, 17 + i, 1e-3) for i, s in enumerate(shapes)]
    bs = [torch.zeros(s, dtype=torch.float32, device=DEV) for s in shapes]
    p2, b2 = [p.clone() for p in ps], [b.clone() for b in bs]
    dm.dmuon_muon_step_batched(ps, gs, bs)
    # any dtype serves as scratch: its size counts in bytes
    ws = torch.empty((dm.dmuon_workspace_bytes(p2) + 3) // 4, dtype=torch.float32, device=DEV)
    dm.dmuon_muon_step_batched_ex(p2, gs, b2, workspace=ws)
    torch.cuda.synchronize()
    for a, b in zip(ps, p2):
        assert torch.equal(a, b)
    for a, b in zip(bs, b2):
        assert torch.equal(a, b)


def test_small_workspace_is_rejected_and_nothing_runs(cuda_lib):
    dm = cuda_lib
    p = _rand((256, 512), torch.bfloat16, 1, 0.02)
    g = _rand((256, 512), torch.bfloat16, 2, 1e-3)
    b = torch.zeros((256, 512), dtype=torch.float32, device=DEV)
    p0 = p.clone()
    ws = torch.empty(1024, dtype=torch.uint8, device=DEV)
    with pytest.raises(dm.DmuonError) as e:
        dm.dmuon_muon_step_batched_ex([p], [g], [b], workspace=ws)
    assert e.value.code == -3
    torch.cuda.synchronize()
    assert torch.equal(p, p0) and torch.count_nonzero(b).item() == 0


def test_allocation_failure_is_reported(cuda_lib):
    dm = cuda_lib
    X = _rand((776, 1552), torch.bfloat16, 3)      # a new size: needs a bigger arena
    dm.dmuon_release_cache()
    dm.dmuon_debug_fail_allocations(1)
    with pytest.raises(dm.DmuonError) as e:
        dm.dmuon_ns_orthogonalize(X, 5)
    assert e.value.code == -3
    dm.dmuon_debug_fail_allocations(0)
    dm.dmuon_ns_orthogonalize(X, 5)                  # works again afterwards
    torch.cuda.synchronize()
    assert dm.dmuon_device_status() == 0


def test_bounded_wait_reports_timeout(cuda_lib):
    """A barrier nothing arrives at: the wait gives up after its limit and the
    device error word says so; the context stays usable."""
    dm = cuda_lib
    assert dm.dmuon_device_status(clear=True) == 0
    dm.dmuon_debug_wait_timeout(2000)
    assert dm.dmuon_device_status(clear=True) == -5
    assert dm.dmuon_device_status() == 0
    X = _rand((128, 256), torch.bfloat16, 4)
    dm.dmuon_ns_orthogonalize(X, 2)
    torch.cuda.synchronize()
    assert dm.dmuon_device_status() == 0


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32], ids=["bf16", "f32"])
def test_update_on_real_weights_is_visible(cuda_lib, dtype):
    """With real (nonzero) weights and an lr large enough that lr X is many
    weight ulps, the change of the weights, W' - W, must match the oracle's
    within the X tolerance: a missing, halved or mis-signed update, or weight
    decay applied twice, fails here (at the bench's lr the update is below half
    a bf16 ulp of most weights, so the weight check alone could not see it)."""
    dm = cuda_lib
    shapes = [(384, 1024), (1200, 264), (256, 256)]
    params = [_rand(s, dtype, 500 + i, 0.02) for i, s in enumerate(shapes)]
    grads = [_rand(s, dtype, 510 + i, 1e-3) for i, s in enumerate(shapes)]
    bufs = [_rand(s, torch.float32, 520 + i, 1e-3) for i, s in enumerate(shapes)]
    W0 = [host(p).astype(np.float64) for p in params]
    g0 = [host(g) for g in grads]
    b0 = [host(b) for b in bufs]
    lr, wd = 0.5, 0.1
    dm.dmuon_muon_step_batched(params, grads, bufs, lr=lr, momentum=0.95, nesterov=True,
                               weight_decay=wd, ns_steps=5)
    torch.cuda.synchronize()
    assert dm.dmuon_device_status() == 0
    for i, s in enumerate(shapes):
        _, X, W_ref = oracle.muon_step(W0[i].astype(np.float32), g0[i], b0[i], lr=lr, momentum=0.95,
                                       nesterov=True, weight_decay=wd, ns_steps=5)
        d_gpu = host(params[i]).astype(np.float64) - W0[i]
        d_ref = W_ref - W0[i]
        # the update is far above the weights' rounding: lr |X| against one ulp of |W|
        assert np.median(np.abs(d_ref)) > 20 * np.median(np.abs(W0[i])) * 2.0 ** -8
        check_rel(d_gpu, d_ref, tol_for(dtype), f"W' - W {s} {dtype}")
