"""fp64 CPU oracle for the batched Muon update (test infrastructure only).

This module is the reference that the CUDA path is checked against.  Only the
tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may
import it; the product path never does.  It shares no code with the CUDA
library: it is a plain, slow restatement of the method in numpy, with one
library primitive (the fp64 matrix product ``@``) as a step.

Sources (page title, section):

* DMuon blog post "DMuon：让矩阵正交化优化器达到接近 AdamW 的分布式训练开销"
  (hankli.space), section "Muon 核心：Newton-Schulz 迭代": normalise
  G0 = G / ||G||_F, then G_{t+1} = 1.5 G_t - 0.5 G_t G_t^T G_t; the code
  listing there transposes when rows > cols, adds 1e-7 to the norm and
  transposes back at the end.
* Same post, section "代码实现 / Vanilla Muon（Baseline，单 GPU）": momentum
  buffer ``buf = momentum * buf + grad`` (multiply, then add), then
  ``p -= lr * update``.
* DMuon training guide "训练指南", section "超参数指南": Nesterov look-ahead
  input is ``grad + momentum * buf``; ``weight_decay`` is a Muon parameter
  (section "第 4 步：创建优化器") without a stated formula.

Readings where the pages are silent:

* Nesterov uses the buffer *after* its update (the update is the first
  statement of the step on the blog's Vanilla Muon).
* Weight decay is decoupled and uses the pre-update weight:
  W' = W (1 - lr wd) - lr X.
* The per-parameter lr scale "0.2 sqrt(max(m, n))" mentioned in the guide's
  hyper-parameter table is off by default (the blog's step uses plain
  ``-lr``); when requested it replaces lr in the whole update, weight decay
  included.
* Gradient clipping (guide, "梯度裁剪") scales every gradient of the call by
  c = min(1, max_norm / (||g|| + 1e-6)) before the momentum update, with the
  2-norm over all of them; the gradient enters as fl32(g * c).
* The transpose test is strict (rows > cols), as in the blog listing.

All pins that tie these functions to the pages and to mathematics live in
``tests/test_oracle_pins.py``.
"""
from __future__ import annotations

import numpy as np

#: Added to the Frobenius norm before dividing (blog, "Muon 核心" code listing).
NORM_EPS = 1e-7
#: Cubic Newton-Schulz coefficients (blog, "Muon 核心", G_{t+1} equation).
NS_A = 1.5
NS_B = -0.5


def momentum_update(buf32: np.ndarray, g32: np.ndarray, mu: float) -> np.ndarray:
    """Momentum buffer ``buf <- mu * buf + g`` in float32.

    Blog, "代码实现 / Vanilla Muon": ``state['buf'].mul_(momentum).add_(grad)``.
    Two separately rounded float32 operations (a product, then a sum), so the
    result is fl32(fl32(mu * buf) + g), with no fused multiply-add.
    """
    buf32 = np.asarray(buf32, dtype=np.float32)
    g32 = np.asarray(g32, dtype=np.float32)
    mu32 = np.float32(mu)
    prod = np.multiply(buf32, mu32, dtype=np.float32)
    return np.add(prod, g32, dtype=np.float32)


def nesterov_input(g32: np.ndarray, buf_new32: np.ndarray, mu: float,
                   nesterov: bool) -> np.ndarray:
    """Input of the orthogonalisation, in fp64.

    Guide, "超参数指南" (nesterov row): ``ns_input = grad + mu * buf`` with the
    already-updated buffer; without Nesterov the input is the buffer itself.
    """
    buf64 = np.asarray(buf_new32, dtype=np.float64)
    if not nesterov:
        return buf64
    return np.asarray(g32, dtype=np.float64) + np.float64(np.float32(mu)) * buf64


def frobenius_normalize(G: np.ndarray) -> np.ndarray:
    """X0 = G / (||G||_F + 1e-7)  (blog, "Muon 核心", G_0 and the listing)."""
    G = np.asarray(G, dtype=np.float64)
    norm = np.sqrt(np.sum(G * G))
    return G / (norm + NORM_EPS)


def ns_iteration(X: np.ndarray, a: float = NS_A, b: float = NS_B, c=None) -> np.ndarray:
    """One Newton-Schulz step.  Cubic: X <- a X + b (X X^T) X; the blog's
    step ("Muon 核心") is a = 1.5, b = -0.5, other (a, b) are the training
    guide's custom coefficients ("超参数指南", ns_backend row).  With a third
    coefficient c the step is the quintic odd polynomial
    X <- a X + b A X + c A^2 X with A = X X^T (the guide's custom
    coefficients read as a degree-5 form)."""
    A = X @ X.T
    if c is None:
        return a * X + b * (A @ X)
    return a * X + b * (A @ X) + c * (A @ (A @ X))


def newton_schulz(G: np.ndarray, steps: int, coeffs=(NS_A, NS_B)) -> np.ndarray:
    """Orthogonalise one 2-D matrix with ``steps`` cubic Newton-Schulz steps.

    Blog, "Muon 核心" listing: transpose when rows > cols, normalise, iterate,
    transpose back.  Returns fp64 with the input's shape.  ``coeffs`` are the
    float32 values (a, b), or (a, b, c) for the quintic form, that the caller
    passes through the C ABI.
    """
    G = np.asarray(G, dtype=np.float64)
    if G.ndim != 2:
        raise ValueError("newton_schulz needs a 2-D matrix")
    if steps < 0:
        raise ValueError("steps must be >= 0")
    if len(coeffs) not in (2, 3):
        raise ValueError("coeffs must be (a, b) or (a, b, c)")
    transposed = G.shape[0] > G.shape[1]
    X = G.T.copy() if transposed else G.copy()
    X = frobenius_normalize(X)
    cf = [float(np.float32(c)) for c in coeffs]
    for _ in range(steps):
        X = ns_iteration(X, *cf)
    return X.T.copy() if transposed else X


def muon_weight_update(W: np.ndarray, X: np.ndarray, lr: float, wd: float) -> np.ndarray:
    """W' = W (1 - lr wd) - lr X in fp64 (blog ``p.add_(update, alpha=-lr)``,
    with decoupled weight decay as read above).  lr and wd are taken as the
    float32 values a caller passes through the C ABI."""
    lr64 = np.float64(np.float32(lr))
    wd64 = np.float64(np.float32(wd))
    return np.asarray(W, dtype=np.float64) * (1.0 - lr64 * wd64) - lr64 * X


def lr_scale_factor(rows: int, cols: int) -> float:
    """Per-parameter lr factor 0.2 sqrt(max(m, n)) (training guide,
    "超参数指南", lr row), as the float32 the library multiplies lr by."""
    return float(np.float32(0.2 * np.sqrt(float(max(rows, cols)))))


def clip_coefficient(grads, max_norm: float):
    """Muon-only global-norm clipping (training guide, "梯度裁剪": global
    p-norm clipping of the Muon gradients before momentum and NS), with p = 2:
    ||g|| over every gradient, c = min(1, max_norm / (||g|| + 1e-6)) rounded
    to float32.  Returns (c, ||g||)."""
    tot = 0.0
    for g in grads:
        g64 = np.asarray(g, dtype=np.float64)
        tot += float(np.sum(g64 * g64))
    norm = float(np.sqrt(tot))
    c = min(1.0, float(np.float32(max_norm)) / (norm + 1e-6))
    return np.float32(c), norm


def round_to_bf16(x32: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (8 significant bits, round to nearest,
    ties to even), returned as the float32 values they widen to exactly.
    bfloat16 is the upper half of the float32 bit pattern, so the rounding is
    done on the integer bits; NaN stays NaN, values past the largest bfloat16
    round to infinity."""
    x32 = np.asarray(x32, dtype=np.float32)
    u = x32.view(np.uint32).astype(np.uint64)
    lsb = (u >> np.uint64(16)) & np.uint64(1)
    r = ((u + np.uint64(0x7FFF) + lsb) >> np.uint64(16)) << np.uint64(16)
    out = r.astype(np.uint32).view(np.float32).copy()
    nan = np.isnan(x32)
    out[nan] = x32[nan]
    return out


def clip_grad_norm_buckets(segments, max_norms):
    """Clipping of several gradient groups ("segments"), each with its own
    norm and coefficient (training guide, "梯度裁剪", the fused
    regular / Muon / AdamW clipping that keeps per-segment semantics).

    ``segments[s]`` is a list of (values, is_bf16) pairs: the gradient values
    as float32 (bfloat16 values widen exactly) and their storage type.  For
    each segment, as for the Muon-only clip: ||g||_s is the 2-norm over all
    of its gradients (fp64), c_s = fl32(min(1, max_norm_s / (||g||_s + 1e-6)))
    with min(1, NaN) = 1, and every gradient becomes fl32(g * c_s), rounded to
    bfloat16 for bfloat16 storage.  Returns (new segments as float32 arrays,
    norms, coefficients)."""
    if len(max_norms) != len(segments):
        raise ValueError("one max_norm per segment")
    out, norms, coefs = [], [], []
    for seg, mx in zip(segments, max_norms):
        c32, nrm = clip_coefficient([v for v, _ in seg], mx)
        new = []
        for v, is_bf16 in seg:
            y = np.multiply(np.asarray(v, np.float32), c32, dtype=np.float32)
            new.append(round_to_bf16(y) if is_bf16 else y)
        out.append(new)
        norms.append(nrm)
        coefs.append(c32)
    return out, norms, coefs


def muon_step(W, g, buf, *, lr: float, momentum: float, nesterov: bool,
              weight_decay: float, ns_steps: int, ns_coeffs=(NS_A, NS_B),
              lr_scale: bool = False, grad_scale=None):
    """One Muon update of one matrix.

    Inputs are numpy arrays: ``W`` and ``g`` as float32 (bf16 values widen
    exactly), ``buf`` float32.  ``grad_scale`` (a float32 clip coefficient)
    makes the gradient enter as fl32(g * c).  ``lr_scale`` multiplies lr by
    0.2 sqrt(max(rows, cols)) in the whole update.  Returns
    ``(buf_new float32, X fp64, W_new fp64)``.
    """
    g32 = np.asarray(g, dtype=np.float32)
    if grad_scale is not None:
        g32 = np.multiply(g32, np.float32(grad_scale), dtype=np.float32)
    buf_new = momentum_update(buf, g32, momentum)
    M = nesterov_input(g32, buf_new, momentum, nesterov)
    X = newton_schulz(M, ns_steps, ns_coeffs)
    lr_eff = lr
    if lr_scale:
        lr_eff = float(np.float32(np.float32(lr) * np.float32(lr_scale_factor(*np.shape(g32)))))
    W_new = muon_weight_update(W, X, lr_eff, weight_decay)
    return buf_new, X, W_new


def orthogonality_error(X: np.ndarray) -> float:
    """||X X^T - I||_F measured on the short side of X.

    Blog, "调试技巧" (check_orthogonality) uses the row Gram; for a tall
    output that Gram is rank-deficient, so the short side is used instead.
    """
    X = np.asarray(X, dtype=np.float64)
    if X.shape[0] > X.shape[1]:
        X = X.T
    R = X @ X.T
    R[np.diag_indices_from(R)] -= 1.0
    return float(np.sqrt(np.sum(R * R)))


def relative_frobenius(a: np.ndarray, b: np.ndarray) -> float:
    """||a - b||_F / ||b||_F (0 when both are zero)."""
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    den = np.sqrt(np.sum(b * b))
    num = np.sqrt(np.sum((a - b) ** 2))
    if den == 0.0:
        return 0.0 if num == 0.0 else float("inf")
    return float(num / den)


def ns_flops(rows: int, cols: int, steps: int, quintic: bool = False) -> float:
    """Useful Newton-Schulz FLOPs of one matrix: per step m^2 n for the
    symmetric product X X^T and 2 m^2 n for (X X^T) X, m = min, n = max;
    the quintic form adds m^3 for the symmetric square A A."""
    m, n = min(rows, cols), max(rows, cols)
    per = 3.0 * m * m * n + (float(m) ** 3 if quintic else 0.0)
    return float(steps) * per


def rank_mean(grads):
    """Data-parallel mean of the ranks' gradients, as the owner computes it
    when it reduces the gradient of a projection it owns (quick start,
    "刚才发生了什么"; blog "参数分片减少 N-S 计算量"): a float32 sum in rank
    order, then one float32 division by the number of ranks (the library's
    fused owner step fixes this order so the buffers are reproducible)."""
    acc = np.array(grads[0], dtype=np.float32, copy=True)
    for g in grads[1:]:
        acc = np.add(acc, np.asarray(g, dtype=np.float32), dtype=np.float32)
    return np.divide(acc, np.float32(len(grads)), dtype=np.float32)


def adamw_step(p, g, m, v, *, lr: float, beta1: float, beta2: float, eps: float,
               weight_decay: float, step: int):
    """AdamW of one tensor (training guide, "第 4 步：创建优化器": the second
    parameter group of dmuon.Muon, with adamw_lr / adamw_betas / adamw_eps /
    adamw_weight_decay; decoupled weight decay, bias-corrected moments).

    The moments follow an exact float32 sequence, c1 = fl32(1 - beta1),
    c2 = fl32(1 - beta2):  m' = fl(fl(beta1 m) + fl(c1 g)),
    v' = fl(fl(beta2 v) + fl(fl(c2 g) g)).  The parameter is computed in fp64:
    p' = p (1 - lr wd) - (lr / bc1) m' / (sqrt(v') / sqrt(bc2) + eps),
    bc1 = 1 - beta1^step, bc2 = 1 - beta2^step.  Returns (m', v', p')."""
    f32 = np.float32
    g32 = np.asarray(g, dtype=np.float32)
    b1, b2 = f32(beta1), f32(beta2)
    c1, c2 = f32(f32(1.0) - b1), f32(f32(1.0) - b2)
    m_new = np.add(np.multiply(np.asarray(m, np.float32), b1, dtype=np.float32),
                   np.multiply(g32, c1, dtype=np.float32), dtype=np.float32)
    v_new = np.add(np.multiply(np.asarray(v, np.float32), b2, dtype=np.float32),
                   np.multiply(np.multiply(g32, c2, dtype=np.float32), g32, dtype=np.float32),
                   dtype=np.float32)
    bc1 = 1.0 - float(b1) ** step
    bc2 = 1.0 - float(b2) ** step
    lr64, wd64, eps64 = float(f32(lr)), float(f32(weight_decay)), float(f32(eps))
    denom = np.sqrt(v_new.astype(np.float64)) / np.sqrt(bc2) + eps64
    p_new = np.asarray(p, np.float64) * (1.0 - lr64 * wd64) - (lr64 / bc1) * m_new.astype(np.float64) / denom
    return m_new, v_new, p_new
