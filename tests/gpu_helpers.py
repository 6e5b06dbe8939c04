"""Helpers shared by the GPU tests: oracle runs on host copies of the same
seeded tensors, and the comparisons with their tolerances.

Tolerances (relative Frobenius error of the orthogonalised X against the fp64
oracle): 2e-2 with bf16 storage, 2e-3 on the fp32 (tf32 operand) path.
Momentum buffers must match bit for bit.  bf16 weights must lie within one
bf16 ulp of the oracle's fp64 weight.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle

TOL_BF16 = 2e-2
TOL_F32 = 2e-3


def host(t: torch.Tensor) -> np.ndarray:
    """Exact host copy (bf16 widens exactly to fp32)."""
    if t.dtype == torch.bfloat16:
        return t.detach().float().cpu().numpy()
    return t.detach().cpu().numpy()


def tol_for(dtype: torch.dtype) -> float:
    return TOL_BF16 if dtype == torch.bfloat16 else TOL_F32


def bf16_ulp(x: np.ndarray) -> np.ndarray:
    """Spacing of bf16 numbers at |x| (8 significant bits)."""
    a = np.abs(np.asarray(x, dtype=np.float64))
    a = np.maximum(a, 2.0 ** -126)
    e = np.floor(np.log2(a))
    return 2.0 ** (e - 7)


def check_bf16_weights(W_gpu: np.ndarray, W_ref: np.ndarray, X_ref: np.ndarray, lr: float,
                       what: str = "W", tol: float = TOL_BF16) -> None:
    """Elementwise: |W_gpu - W_ref| <= 1 bf16 ulp (at the larger of the two)
    + lr * tol * max|X_ref|.  The second term is the update error that the X
    tolerance allows; it matters only where W' cancels to near zero, where
    one ulp of W' is far below any error of lr * X."""
    ulp = np.maximum(bf16_ulp(W_ref), bf16_ulp(W_gpu))
    slack = float(lr) * tol * float(np.max(np.abs(X_ref)))
    err = np.abs(W_gpu.astype(np.float64) - W_ref)
    bad = err > ulp * (1.0 + 1e-6) + slack
    assert not bad.any(), (f"{what}: {int(bad.sum())} of {bad.size} elements beyond 1 bf16 ulp "
                           f"+ {slack:.2e}; worst {float(((err - slack) / ulp).max()):.2f} ulp")


def check_rel(got: np.ndarray, want: np.ndarray, tol: float, what: str) -> float:
    r = oracle.relative_frobenius(got, want)
    assert r <= tol, f"{what}: relative Frobenius error {r:.3e} > {tol:.1e}"
    return r


def oracle_step(W, g, buf, *, lr, momentum, nesterov, weight_decay, ns_steps):
    return oracle.muon_step(host(W), host(g), host(buf), lr=lr, momentum=momentum,
                            nesterov=nesterov, weight_decay=weight_decay, ns_steps=ns_steps)
