"""Seeded synthetic workloads for the batched Muon update.

This module only draws inputs (weights, gradients, momentum buffers and
matrix shapes).  It holds none of the update's arithmetic, so the tests can
feed the very same tensors to the CUDA path and to the fp64 oracle.

The shapes follow the pages' workloads:

* ``fp32_256x512``: one 256x512 fp32 matrix.
* ``tinymlp``: the quick-start TinyMLP (DMuon docs "快速开始", model.py):
  d=512, ff=2048, 4 layers of gate/up (2048x512) and down (512x2048).
* ``square4096``: one 4096x4096 projection, the size the DMuon blog post uses
  in its time-split table ("分布式 Muon 的性能瓶颈").
* ``llama8b``: 32 Llama-8B-style layers (q/o 4096x4096, k/v 1024x4096,
  gate/up 14336x4096, down 4096x14336); the projection names are those the
  DMuon training guide routes to Muon ("高级模式：Type-Split Routing").
* ``mixed1024``: 1024 matrices with power-of-two sides in [128, 8192] and
  aspect ratio <= 16, half with Student-t(3) gradients, half rank-8 plus
  small noise (small GateDelta-style projections next to large FFNs, as the
  guide's predicate examples describe).
"""
from __future__ import annotations

import dataclasses
import math
from typing import List, Optional, Sequence

import numpy as np
import torch


@dataclasses.dataclass(frozen=True)
class MatrixSpec:
    name: str
    rows: int
    cols: int
    grad_kind: str = "gaussian"   # gaussian | student_t3 | rank8

    @property
    def numel(self) -> int:
        return self.rows * self.cols


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    dtype: torch.dtype            # parameter and gradient dtype
    specs: Sequence[MatrixSpec]
    grad_std: float
    lr: float = 0.02
    momentum: float = 0.95
    nesterov: bool = True
    weight_decay: float = 0.0
    ns_steps: int = 5
    seed: int = 0
    w_std: float = 0.02
    prior_steps: int = 0          # momentum history: steps run before the measured one

    @property
    def numel(self) -> int:
        return sum(s.numel for s in self.specs)


def _tinymlp_specs() -> List[MatrixSpec]:
    specs = []
    for layer in range(4):
        specs.append(MatrixSpec(f"layers.{layer}.gate_proj", 2048, 512))
        specs.append(MatrixSpec(f"layers.{layer}.up_proj", 2048, 512))
        specs.append(MatrixSpec(f"layers.{layer}.down_proj", 512, 2048))
    return specs


def _llama8b_specs(layers: int = 32) -> List[MatrixSpec]:
    specs = []
    for layer in range(layers):
        p = f"layers.{layer}."
        specs += [
            MatrixSpec(p + "q_proj", 4096, 4096),
            MatrixSpec(p + "k_proj", 1024, 4096),
            MatrixSpec(p + "v_proj", 1024, 4096),
            MatrixSpec(p + "o_proj", 4096, 4096),
            MatrixSpec(p + "gate_proj", 14336, 4096),
            MatrixSpec(p + "up_proj", 14336, 4096),
            MatrixSpec(p + "down_proj", 4096, 14336),
        ]
    return specs


def mixed_shapes(count: int = 1024, seed: int = 4) -> List[MatrixSpec]:
    """Power-of-two sides in {128..8192}, drawn i.i.d., aspect ratio <= 16
    (pairs beyond it are redrawn); even indices Student-t(3) gradients, odd
    indices rank-8 plus noise."""
    rng = np.random.default_rng(seed)
    sides = [128 << i for i in range(7)]
    specs = []
    while len(specs) < count:
        r, c = (int(v) for v in rng.choice(sides, size=2))
        if max(r, c) > 16 * min(r, c):
            continue
        i = len(specs)
        kind = "student_t3" if i % 2 == 0 else "rank8"
        specs.append(MatrixSpec(f"mixed.{i}", r, c, kind))
    return specs


def workload(name: str) -> Workload:
    """The named synthetic workload."""
    if name == "fp32_256x512":
        return Workload(name, torch.float32, [MatrixSpec("w", 256, 512)], grad_std=1.0, seed=0)
    if name == "tinymlp":
        return Workload(name, torch.bfloat16, _tinymlp_specs(), grad_std=1e-3, seed=1,
                        prior_steps=3)
    if name == "square4096":
        return Workload(name, torch.bfloat16, [MatrixSpec("proj", 4096, 4096)], grad_std=1e-3,
                        weight_decay=0.01, seed=2)
    if name == "llama8b":
        return Workload(name, torch.bfloat16, _llama8b_specs(), grad_std=1e-4, seed=3)
    if name == "llama8b_layer":
        # one layer of the stack: the small case for profiler captures
        return Workload(name, torch.bfloat16, _llama8b_specs(1), grad_std=1e-4, seed=3)
    if name == "mixed1024":
        return Workload(name, torch.bfloat16, mixed_shapes(), grad_std=1.0, seed=4)
    raise KeyError(name)


WORKLOADS = ("fp32_256x512", "tinymlp", "square4096", "llama8b", "mixed1024", "llama8b_layer")


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _draw_grad(spec: MatrixSpec, std: float, dtype, device, gen) -> torch.Tensor:
    shape = (spec.rows, spec.cols)
    if spec.grad_kind == "gaussian":
        t = torch.empty(shape, dtype=torch.float32, device=device).normal_(0.0, std, generator=gen)
    elif spec.grad_kind == "student_t3":
        # Student-t with 3 degrees of freedom, unit scale: Z / sqrt(chi2_3 / 3).
        z = torch.empty(shape, dtype=torch.float32, device=device).normal_(generator=gen)
        chi = torch.zeros(shape, dtype=torch.float32, device=device)
        for _ in range(3):
            e = torch.empty(shape, dtype=torch.float32, device=device).normal_(generator=gen)
            chi.addcmul_(e, e)
        t = z / torch.sqrt(chi / 3.0)
        del z, chi
    elif spec.grad_kind == "rank8":
        u = torch.empty((spec.rows, 8), dtype=torch.float32, device=device).normal_(generator=gen)
        v = torch.empty((spec.cols, 8), dtype=torch.float32, device=device).normal_(generator=gen)
        t = (u @ v.T) * (1e-3 / math.sqrt(8.0))
        t += torch.empty(shape, dtype=torch.float32, device=device).normal_(0.0, 1e-6, generator=gen)
    else:
        raise ValueError(spec.grad_kind)
    return t.to(dtype)


@dataclasses.dataclass
class Tensors:
    params: List[torch.Tensor]
    grads: List[torch.Tensor]
    bufs: List[torch.Tensor]
    prior_grads: List[List[torch.Tensor]]   # [step][matrix], empty unless prior_steps > 0
    flat: Optional[tuple] = None             # (params, grads, bufs) flat storage when drawn flat


def make_tensors(wl: Workload, device="cpu", subset: Optional[Sequence[int]] = None,
                 draw_grads: bool = True, flat: bool = False, seed_offset: int = 0) -> Tensors:
    """Draw the workload's tensors on ``device``.

    Every matrix gets its own generator seeded from (workload seed, index), so
    a subset draws exactly the tensors the full workload would.  Momentum
    buffers start at zero; workloads with a momentum history carry
    ``prior_steps`` extra gradient sets to be applied first.  ``flat`` places
    each kind (weights, gradients, buffers) in one contiguous allocation, the
    matrices being views into it; ``seed_offset`` draws an independent copy.
    """
    idx = list(range(len(wl.specs))) if subset is None else list(subset)
    params, grads, bufs = [], [], []
    prior = [[] for _ in range(wl.prior_steps)]
    if flat:
        tot = sum(wl.specs[i].numel for i in idx)
        pflat = torch.empty(tot, dtype=wl.dtype, device=device)
        gflat = torch.empty(tot, dtype=wl.dtype, device=device) if draw_grads else None
        bflat = torch.zeros(tot, dtype=torch.float32, device=device)
    off = 0
    for i in idx:
        spec = wl.specs[i]
        shape = (spec.rows, spec.cols)
        gen = _gen(wl.seed * 1_000_003 + i + 7_919 * seed_offset, device)
        w = torch.empty(shape, dtype=torch.float32, device=device)
        w.normal_(0.0, wl.w_std, generator=gen)
        if flat:
            params.append(pflat[off:off + spec.numel].view(shape))
            params[-1].copy_(w)
        else:
            params.append(w.to(wl.dtype))
        del w
        for s in range(wl.prior_steps):
            prior[s].append(_draw_grad(spec, wl.grad_std, wl.dtype, device, gen))
        if draw_grads:
            g = _draw_grad(spec, wl.grad_std, wl.dtype, device, gen)
            if flat:
                grads.append(gflat[off:off + spec.numel].view(shape))
                grads[-1].copy_(g)
                del g
            else:
                grads.append(g)
        if flat:
            bufs.append(bflat[off:off + spec.numel].view(shape))
        else:
            bufs.append(torch.zeros(shape, dtype=torch.float32, device=device))
        off += spec.numel
    t = Tensors(params, grads, bufs, prior)
    if flat:
        t.flat = (pflat, gflat, bflat)
    return t


def ns_flops(wl: Workload, steps: Optional[int] = None) -> float:
    """Useful Newton-Schulz FLOPs of one step over the workload: per NS step
    m^2 n for X X^T plus 2 m^2 n for (X X^T) X, with m = min(rows, cols)."""
    k = wl.ns_steps if steps is None else steps
    tot = 0.0
    for s in wl.specs:
        m, n = min(s.rows, s.cols), max(s.rows, s.cols)
        tot += 3.0 * m * m * n * k
    return tot
