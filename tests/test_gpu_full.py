"""Full-size workloads, in the launch configuration bench.py times (needs a B200).

* square4096: one 4096 x 4096 bf16 projection (weight decay 0.01), one Muon
  step, and the step-count sweep k = 3, 5, 7, 10 with the orthogonality error
  ||X X^T - I||_F of the GPU result next to the oracle's.
* llama8b: the whole 224-matrix Llama-8B-shaped stack in one batched call.
* mixed1024: 1024 mixed-shape matrices (Student-t and rank-8 gradients).

For the two batches the GPU runs every matrix in one call; the fp64 oracle then
recomputes a sample of them one by one.  Their weights start at zero, so the
updated weight is bf16(-lr X) and shows the orthogonalised matrix itself at
bf16 precision; the momentum buffers are compared bit for bit.
"""
import numpy as np
import pytest
import torch

import oracle
from newton_schulz_09_b200 import synthetic
from tests.gpu_helpers import TOL_BF16, check_bf16_weights, check_rel, host

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def test_square4096_step(cuda_lib):
    dm = cuda_lib
    wl = synthetic.workload("square4096")
    t = synthetic.make_tensors(wl, device=DEV)
    W0, g, b0 = host(t.params[0]), host(t.grads[0]), host(t.bufs[0])
    Wz = torch.zeros_like(t.params[0])
    bz = t.bufs[0].clone()
    dm.dmuon_muon_step_batched([t.params[0], Wz], [t.grads[0], t.grads[0].clone()], [t.bufs[0], bz],
                               lr=wl.lr, momentum=wl.momentum, nesterov=wl.nesterov,
                               weight_decay=wl.weight_decay, ns_steps=wl.ns_steps)
    torch.cuda.synchronize()
    assert dm.dmuon_device_status() == 0
    buf_ref, X_ref, W_ref = oracle.muon_step(W0, g, b0, lr=wl.lr, momentum=wl.momentum,
                                             nesterov=wl.nesterov, weight_decay=wl.weight_decay,
                                             ns_steps=wl.ns_steps)
    assert np.array_equal(host(t.bufs[0]).view(np.uint32), buf_ref.view(np.uint32))
    assert np.array_equal(host(bz).view(np.uint32), buf_ref.view(np.uint32))
    lr = float(np.float32(wl.lr))
    check_rel(host(Wz), -lr * X_ref, TOL_BF16, "square4096 -lr X")
    check_bf16_weights(host(t.params[0]), W_ref, X_ref, wl.lr, "square4096 W")


def test_square4096_step_sweep(cuda_lib):
    """Orthogonality error of the GPU result for k = 3, 5, 7, 10 (the sweep of
    the blog's debugging section) against the oracle's."""
    dm = cuda_lib
    wl = synthetic.workload("square4096")
    t = synthetic.make_tensors(wl, device=DEV)
    G = t.grads[0]
    X = oracle.frobenius_normalize(host(G))
    prev = None
    done = 0
    for k in (3, 5, 7, 10):
        for _ in range(k - done):
            X = oracle.ns_iteration(X)
        done = k
        Y = G.clone()
        dm.dmuon_ns_orthogonalize(Y, k)
        torch.cuda.synchronize()
        Yh = host(Y).astype(np.float64)
        check_rel(Yh, X, TOL_BF16, f"square4096 NS k={k}")
        e_gpu, e_ref = oracle.orthogonality_error(Yh), oracle.orthogonality_error(X)
        print(f"k={k}: ||XX^T - I||_F gpu {e_gpu:.4f} oracle {e_ref:.4f}")
        assert abs(e_gpu - e_ref) <= 2e-2 * e_ref
        if prev is not None:
            assert e_ref <= prev
        prev = e_ref


def _batched_zero_weight_step(dm, wl, sample):
    t = synthetic.make_tensors(wl, device=DEV, flat=True)
    for p in t.params:
        p.zero_()
    gs = {i: host(t.grads[i]) for i in sample}
    dm.dmuon_muon_step_batched(t.params, t.grads, t.bufs, lr=wl.lr, momentum=wl.momentum,
                               nesterov=wl.nesterov, weight_decay=wl.weight_decay,
                               ns_steps=wl.ns_steps)
    torch.cuda.synchronize()
    assert dm.dmuon_device_status() == 0
    lr = float(np.float32(wl.lr))
    for i in sample:
        buf_ref, X_ref, _ = oracle.muon_step(np.zeros(gs[i].shape, np.float32), gs[i],
                                             np.zeros(gs[i].shape, np.float32), lr=wl.lr,
                                             momentum=wl.momentum, nesterov=wl.nesterov,
                                             weight_decay=wl.weight_decay, ns_steps=wl.ns_steps)
        spec = wl.specs[i]
        assert np.array_equal(host(t.bufs[i]).view(np.uint32), buf_ref.view(np.uint32)), spec
        r = check_rel(host(t.params[i]), -lr * X_ref, TOL_BF16, f"{wl.name}[{i}] {spec.rows}x{spec.cols}")
        print(f"{spec.name} {spec.rows}x{spec.cols}: rel err {r:.2e}")
    del t
    torch.cuda.empty_cache()


@pytest.mark.slow
def test_llama8b_full_batch_sampled(cuda_lib):
    wl = synthetic.workload("llama8b")
    # layer 0: q, k, v, o, gate (tall), down (wide); layer 31: k
    sample = [0, 1, 2, 3, 4, 6, 7 * 31 + 1]
    _batched_zero_weight_step(cuda_lib, wl, sample)


@pytest.mark.slow
def test_mixed1024_full_batch_sampled(cuda_lib):
    wl = synthetic.workload("mixed1024")
    fl = [3.0 * min(s.rows, s.cols) ** 2 * max(s.rows, s.cols) for s in wl.specs]
    rng = np.random.default_rng(5)
    small = [i for i, s in enumerate(wl.specs) if s.rows * s.cols <= (1 << 20)]
    sample = sorted(rng.choice(small, size=min(24, len(small)), replace=False).tolist())
    # the four largest matrices the oracle handles in seconds
    big = sorted((i for i in range(len(fl)) if fl[i] <= 6e11), key=lambda i: -fl[i])
    for i in big:
        if len(sample) >= 28:
            break
        if i not in sample:
            sample.append(i)
    kinds = {wl.specs[i].grad_kind for i in sample}
    assert kinds == {"student_t3", "rank8"}
    assert any(wl.specs[i].rows > wl.specs[i].cols for i in sample)
    assert any(wl.specs[i].rows < wl.specs[i].cols for i in sample)
    _batched_zero_weight_step(cuda_lib, wl, sample)
