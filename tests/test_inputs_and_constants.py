"""Synthetic inputs and page constants (CPU only)."""
import os

import numpy as np
import torch

import oracle
from newton_schulz_09_b200 import synthetic

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "pages_constants.txt")


def _constants():
    out = {}
    with open(GOLDEN) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            k, *v = line.split()
            out[k] = [float(x) for x in v]
    return out


def test_oracle_uses_page_constants():
    c = _constants()
    assert oracle.NS_A == c["ns_coeff_a"][0]
    assert oracle.NS_B == c["ns_coeff_b"][0]
    assert oracle.NORM_EPS == c["norm_eps"][0]


def test_workloads_use_page_defaults():
    c = _constants()
    for name in synthetic.WORKLOADS:
        wl = synthetic.workload(name)
        assert wl.lr == c["lr"][0]
        assert wl.momentum == c["momentum"][0]
        assert wl.ns_steps == c["ns_steps"][0]
        assert wl.nesterov == bool(c["nesterov"][0])
    tm = synthetic.workload("tinymlp")
    d, ff = int(c["tinymlp_d"][0]), int(c["tinymlp_ff"][0])
    assert len(tm.specs) == 3 * int(c["tinymlp_layers"][0])
    assert {(s.rows, s.cols) for s in tm.specs} == {(ff, d), (d, ff)}


def test_llama_stack_shapes():
    wl = synthetic.workload("llama8b")
    assert len(wl.specs) == 224
    assert wl.numel == 32 * (2 * 4096 * 4096 + 2 * 1024 * 4096 + 3 * 14336 * 4096)
    assert abs(synthetic.ns_flops(wl) - 4.164e14) / 4.164e14 < 1e-3


def test_mixed_shapes():
    specs = synthetic.mixed_shapes()
    assert len(specs) == 1024
    sides = {128 << i for i in range(7)}
    for s in specs:
        assert s.rows in sides and s.cols in sides
        assert max(s.rows, s.cols) <= 16 * min(s.rows, s.cols)
    assert {s.grad_kind for s in specs[0::2]} == {"student_t3"}
    assert {s.grad_kind for s in specs[1::2]} == {"rank8"}
    assert any(s.rows > s.cols for s in specs) and any(s.rows < s.cols for s in specs)
    assert specs == synthetic.mixed_shapes()


def test_generator_is_seeded_and_subsettable():
    wl = synthetic.workload("tinymlp")
    a = synthetic.make_tensors(wl)
    b = synthetic.make_tensors(wl, subset=[4, 7])
    assert torch.equal(a.params[4], b.params[0]) and torch.equal(a.grads[7], b.grads[1])
    assert len(a.prior_grads) == 3 and torch.equal(a.prior_grads[2][7], b.prior_grads[2][1])
    assert a.params[0].dtype == torch.bfloat16 and a.bufs[0].dtype == torch.float32
    g = a.grads[0].float()
    assert abs(g.std().item() - 1e-3) < 1e-4


def test_grad_kinds_have_their_structure():
    wl = synthetic.Workload("t", torch.bfloat16,
                            [synthetic.MatrixSpec("a", 256, 512, "rank8"),
                             synthetic.MatrixSpec("b", 256, 512, "student_t3")], grad_std=1.0)
    t = synthetic.make_tensors(wl)
    s = np.linalg.svd(t.grads[0].float().numpy().astype(np.float64), compute_uv=False)
    assert s[7] > 100 * s[8]                       # rank 8 plus small noise
    x = t.grads[1].float().numpy()
    kurt = np.mean(x ** 4) / np.mean(x ** 2) ** 2
    assert kurt > 6.0                              # heavy tails (Gaussian: 3)
