"""The GEMM stage on CTA pairs (256 x 256 tiles, pair UMMAs) against the
oracle (needs a B200).  Groups of bf16 matrices with m % 256 == 0 whose SYRK
runs on 256 x 256 tiles take this kernel; each case first checks that the
plan chose it, then compares the update with the oracle's Muon step on the
same inputs.  Cases: one square matrix (first, middle and last GEMM steps),
a batch with transposed (tall) parameters, column counts that end inside a
pair tile's second half (n % 256 == 64 and 192), Nesterov off with weight
decay on real weights, one Newton-Schulz step (the first GEMM is the
last), and the quintic coefficients."""
import numpy as np
import pytest
import torch

import oracle
from tests.gpu_helpers import TOL_BF16, check_bf16_weights, check_rel, host

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _rand(shape, dtype, seed, std=1.0):
    g = torch.Generator(device=DEV)
    g.manual_seed(seed)
    return (torch.randn(shape, generator=g, device=DEV) * std).to(dtype)


def _run(dm, shapes, *, seed, ns_steps, zero_w=True, nesterov=True, wd=0.0, lr=0.05, coeffs=None):
    params = [torch.zeros(s, dtype=torch.bfloat16, device=DEV) if zero_w
              else _rand(s, torch.bfloat16, seed + 100 + i, 0.02) for i, s in enumerate(shapes)]
    w0 = [host(p) for p in params]
    grads = [_rand(s, torch.bfloat16, seed + i, 1e-3) for i, s in enumerate(shapes)]
    bufs = [_rand(s, torch.float32, seed + 50 + i, 1e-3) for i, s in enumerate(shapes)]
    b0 = [host(b) for b in bufs]
    if coeffs is None:
        dm.dmuon_muon_step_batched(params, grads, bufs, lr=lr, momentum=0.95, nesterov=nesterov,
                                   weight_decay=wd, ns_steps=ns_steps)
    else:
        dm.dmuon_muon_step_batched_opts(params, grads, bufs, lr=lr, momentum=0.95, nesterov=nesterov,
                                        weight_decay=wd, ns_steps=ns_steps, ns_coefficients=coeffs)
    torch.cuda.synchronize()
    assert dm.dmuon_device_status() == 0
    plan = dm.dmuon_debug_last_plan()
    assert plan and all(g["gemm_pair"] and g["syrk256"] for g in plan), plan
    if coeffs is not None and len(coeffs) == 3:
        # the SQUARE on 256 x 256 tiles wherever A has its 3-D view (m % 64 == 0)
        want = all(min(s) % 64 == 0 for s in shapes)
        assert all(g["square256"] == want for g in plan), plan
    for i, s in enumerate(shapes):
        buf_ref, X_ref, W_ref = oracle.muon_step(w0[i], host(grads[i]), b0[i], lr=lr, momentum=0.95,
                                                 nesterov=nesterov, weight_decay=wd, ns_steps=ns_steps,
                                                 ns_coeffs=coeffs or (1.5, -0.5))
        assert np.array_equal(host(bufs[i]).view(np.uint32), buf_ref.view(np.uint32))
        if zero_w and wd == 0.0:
            check_rel(host(params[i]), W_ref, TOL_BF16, f"pair GEMM {s} k={ns_steps}")
        else:
            check_bf16_weights(host(params[i]), W_ref, X_ref, lr, f"pair GEMM {s} k={ns_steps}")


@pytest.mark.slow
def test_square_4096(cuda_lib):
    # 16 x 16 pair tiles; steps 1..3 run the first, a middle and the last GEMM
    _run(cuda_lib, [(4096, 4096)], seed=300, ns_steps=3)


def test_batch_with_tall_matrices(cuda_lib):
    # m = 1024 everywhere: four 1024 x 4096, two 4096 x 1024 (transposed),
    # two 1024 x 2048 -- enough SYRK tiles for the 256 x 256 kernel
    shapes = [(1024, 4096)] * 4 + [(4096, 1024)] * 2 + [(1024, 2048)] * 2
    _run(cuda_lib, shapes, seed=310, ns_steps=2)


@pytest.mark.parametrize("n", [4160, 3264], ids=["n%256=64", "n%256=192"])
def test_columns_ending_inside_a_pair_tile(cuda_lib, n):
    # the last pair tile's second CTA gets 0 or 64 of its 128 X columns
    shapes = [(1024, n)] * 6 + [(n, 1024)] * 2
    _run(cuda_lib, shapes, seed=320, ns_steps=2)


def test_weight_decay_without_nesterov(cuda_lib):
    shapes = [(512, 2048)] * 26 + [(2048, 512)] * 4
    _run(cuda_lib, shapes, seed=330, ns_steps=3, zero_w=False, nesterov=False, wd=0.1, lr=0.02)


def test_one_step(cuda_lib):
    shapes = [(768, 3072)] * 14
    _run(cuda_lib, shapes, seed=340, ns_steps=1)


def test_quintic_coefficients(cuda_lib):
    # P = b A + c A A from the SQUARE stage, which reads A's upper triangle
    # (lower k-blocks transposed) and stores P's diagonal 256-blocks whole for
    # the pair GEMM
    shapes = [(1024, 4096)] * 4 + [(4096, 1024)] * 2 + [(1024, 2048)] * 2
    _run(cuda_lib, shapes, seed=350, ns_steps=3, coeffs=(3.4445, -4.7750, 2.0315))


@pytest.mark.parametrize("shapes", [
    [(384, 1536)] * 36 + [(1536, 384)] * 4,      # m % 256 == 128: the last pair's odd CTA holds no rows
    [(1000, 3008)] * 8 + [(3008, 1000)] * 2,     # ragged m: the last pair's odd CTA holds 104 rows
], ids=["m%256=128", "m=1000"])
def test_rows_ending_inside_a_pair_tile(cuda_lib, shapes):
    _run(cuda_lib, shapes, seed=360, ns_steps=2)


@pytest.mark.parametrize("shapes", [
    [(384, 1536)] * 36 + [(1536, 384)] * 4,
    [(1000, 3008)] * 8 + [(3008, 1000)] * 2,
], ids=["m%256=128", "m=1000"])
def test_quintic_rows_ending_inside_a_pair_tile(cuda_lib, shapes):
    # the SQUARE stage reads A's k-blocks left of each operand's diagonal
    # 256-block transposed, with the last column band partly past m
    _run(cuda_lib, shapes, seed=370, ns_steps=2, coeffs=(3.4445, -4.7750, 2.0315))
