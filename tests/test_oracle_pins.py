"""The oracle against facts the pages and mathematics fix (CPU only).

Each pin in ``tests/pins.py`` runs on the oracle and must hold.  The
mutation tests then plant one plausible mistake at a time in a copy of the
oracle (on the CPU) and check that at least one pin catches it, which is what
makes the pins worth trusting.
"""
import types

import numpy as np
import pytest

import oracle
from oracle import muon_oracle
from tests import pins


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=lambda p: p.__name__)
def test_pin_holds(pin):
    pin(oracle)


def test_jacobi_svd_matches_lapack():
    rng = np.random.default_rng(3)
    for shape in ((5, 9), (9, 5), (16, 16)):
        G = rng.standard_normal(shape)
        U, s, V = pins.jacobi_svd(G)
        assert np.allclose((U * s) @ V.T, G, atol=1e-13)
        assert np.allclose(np.sort(s)[::-1], np.linalg.svd(G, compute_uv=False), atol=1e-13)


def test_exact_rounding_helper():
    from fractions import Fraction
    assert pins.exact_f32_round(Fraction(1, 3)) == np.float32(1.0 / 3.0)
    # 1 + 2^-24 is a tie between 1 and 1 + 2^-23: ties to even gives 1
    assert pins.exact_f32_round(Fraction(1) + Fraction(1, 2 ** 24)) == np.float32(1.0)


def _mutant(**overrides):
    """A copy of the oracle module with some functions or constants replaced."""
    m = types.ModuleType("mutant_oracle")
    for k in dir(muon_oracle):
        if not k.startswith("__"):
            setattr(m, k, getattr(muon_oracle, k))
    for k, v in overrides.items():
        setattr(m, k, v)
    # rebind the module-level helpers so that replaced pieces are used
    def newton_schulz(G, steps, coeffs=(1.5, -0.5)):
        G = np.asarray(G, dtype=np.float64)
        transposed = G.shape[0] > G.shape[1]
        X = G.T.copy() if transposed else G.copy()
        X = m.frobenius_normalize(X)
        cf = [float(np.float32(c)) for c in coeffs]
        for _ in range(steps):
            X = m.ns_iteration(X, *cf)
        return X.T.copy() if transposed else X

    def muon_step(W, g, buf, *, lr, momentum, nesterov, weight_decay, ns_steps,
                  ns_coeffs=(1.5, -0.5), lr_scale=False, grad_scale=None):
        g32 = np.asarray(g, dtype=np.float32)
        if grad_scale is not None:
            g32 = np.multiply(g32, np.float32(grad_scale), dtype=np.float32)
        buf_new = m.momentum_update(buf, g32, momentum)
        M = m.nesterov_input(g32, buf_new, momentum, nesterov)
        X = m.newton_schulz(M, ns_steps, ns_coeffs)
        lr_eff = lr
        if lr_scale:
            lr_eff = float(np.float32(np.float32(lr) * np.float32(m.lr_scale_factor(*np.shape(g32)))))
        return buf_new, X, m.muon_weight_update(W, X, lr_eff, weight_decay)

    if "newton_schulz" not in overrides:
        m.newton_schulz = newton_schulz
    if "muon_step" not in overrides:
        m.muon_step = muon_step
    return m


def _no_eps(G):
    G = np.asarray(G, dtype=np.float64)
    n = np.sqrt(np.sum(G * G))
    return G / n if n > 0 else G


MUTANTS = {
    "sign_of_cubic_term": dict(ns_iteration=lambda X, a=1.5, b=-0.5, c=None: a * X - b * (X @ X.T) @ X + (0 if c is None else c * (X @ X.T) @ ((X @ X.T) @ X))),
    "coefficient_3_not_1.5": dict(ns_iteration=lambda X, a=1.5, b=-0.5, c=None: 2 * a * X + b * (X @ X.T) @ X + (0 if c is None else c * (X @ X.T) @ ((X @ X.T) @ X))),
    # X^T X in place of X X^T: only expressible for square X (otherwise the
    # shapes do not conform), where it differs unless X is normal.
    "gram_of_columns": dict(ns_iteration=lambda X, a=1.5, b=-0.5, c=None: a * X + b * ((X.T @ X) @ X if X.shape[0] == X.shape[1] else (X @ X.T) @ X)),
    "one_step_short": dict(ns_iteration=lambda X, a=1.5, b=-0.5, c=None: X),
    "dropped_norm_eps": dict(frobenius_normalize=_no_eps),
    "eps_on_squared_norm": dict(frobenius_normalize=lambda G: np.asarray(G, np.float64) / np.sqrt(np.sum(np.asarray(G, np.float64) ** 2) + 1e-7)),
    "no_normalisation": dict(frobenius_normalize=lambda G: np.asarray(G, np.float64)),
    "fma_momentum": dict(momentum_update=lambda b, g, mu: (np.float64(np.float32(mu)) * np.asarray(b, np.float64) + np.asarray(g, np.float64)).astype(np.float32)),
    "lerp_momentum": dict(momentum_update=lambda b, g, mu: (np.float32(mu) * np.asarray(b, np.float32) + np.float32(1 - mu) * np.asarray(g, np.float32)).astype(np.float32)),
    "nesterov_pre_update": dict(),   # filled below
    "weight_decay_sign": dict(muon_weight_update=lambda W, X, lr, wd: np.asarray(W, np.float64) * (1.0 + float(np.float32(lr)) * float(np.float32(wd))) - float(np.float32(lr)) * X),
    "update_sign": dict(muon_weight_update=lambda W, X, lr, wd: np.asarray(W, np.float64) * (1.0 - float(np.float32(lr)) * float(np.float32(wd))) + float(np.float32(lr)) * X),
}


def _pre_update_step(W, g, buf, *, lr, momentum, nesterov, weight_decay, ns_steps,
                     ns_coeffs=(1.5, -0.5), lr_scale=False, grad_scale=None):
    g32 = np.asarray(g, dtype=np.float32)
    if grad_scale is not None:
        g32 = np.multiply(g32, np.float32(grad_scale), dtype=np.float32)
    M = muon_oracle.nesterov_input(g32, buf, momentum, nesterov)       # old buffer
    buf_new = muon_oracle.momentum_update(buf, g32, momentum)
    X = muon_oracle.newton_schulz(M, ns_steps, ns_coeffs)
    lr_eff = lr
    if lr_scale:
        lr_eff = float(np.float32(np.float32(lr) * np.float32(muon_oracle.lr_scale_factor(*np.shape(g32)))))
    return buf_new, X, muon_oracle.muon_weight_update(W, X, lr_eff, weight_decay)


MUTANTS["nesterov_pre_update"] = dict(muon_step=_pre_update_step)


def _clip_after_momentum(W, g, buf, *, lr, momentum, nesterov, weight_decay, ns_steps,
                         ns_coeffs=(1.5, -0.5), lr_scale=False, grad_scale=None):
    buf_new = muon_oracle.momentum_update(buf, g, momentum)
    if grad_scale is not None:
        buf_new = np.multiply(buf_new, np.float32(grad_scale), dtype=np.float32)
    M = muon_oracle.nesterov_input(g, buf_new, momentum, nesterov)
    X = muon_oracle.newton_schulz(M, ns_steps, ns_coeffs)
    return buf_new, X, muon_oracle.muon_weight_update(W, X, lr, weight_decay)


def _lr_scale_min_side(W, g, buf, **kw):
    if kw.get("lr_scale"):
        kw = dict(kw)
        kw["lr_scale"] = False
        kw["lr"] = float(np.float32(kw["lr"] * 0.2 * np.sqrt(min(np.shape(g)))))
    return muon_oracle.muon_step(W, g, buf, **kw)


def _coeffs_ignored(G, steps, coeffs=(1.5, -0.5)):
    return muon_oracle.newton_schulz(G, steps)


def _adamw_variant(kind):
    def step_fn(p, g, m, v, *, lr, beta1, beta2, eps, weight_decay, step):
        f32 = np.float32
        g32 = np.asarray(g, np.float32)
        if kind == "l2_decay":
            g32 = (g32 + f32(weight_decay) * np.asarray(p, np.float32)).astype(np.float32)
        m_new = (f32(beta1) * np.asarray(m, np.float32) + (f32(1) - f32(beta1)) * g32).astype(np.float32)
        v_new = (f32(beta2) * np.asarray(v, np.float32) + (f32(1) - f32(beta2)) * g32 * g32).astype(np.float32)
        bc1 = 1.0 - float(f32(beta1)) ** step if kind != "no_bias_correction" else 1.0
        bc2 = 1.0 - float(f32(beta2)) ** step if kind != "no_bias_correction" else 1.0
        if kind == "eps_inside_sqrt":
            denom = np.sqrt(v_new.astype(np.float64) / bc2 + float(f32(eps)))
        else:
            denom = np.sqrt(v_new.astype(np.float64)) / np.sqrt(bc2) + float(f32(eps))
        wd = 0.0 if kind == "l2_decay" else float(f32(weight_decay))
        p_new = np.asarray(p, np.float64) * (1.0 - float(f32(lr)) * wd) - (float(f32(lr)) / bc1) * m_new / denom
        return m_new, v_new, p_new
    return step_fn


MUTANTS["adamw_no_bias_correction"] = dict(adamw_step=_adamw_variant("no_bias_correction"))
MUTANTS["adamw_l2_decay"] = dict(adamw_step=_adamw_variant("l2_decay"))
MUTANTS["adamw_eps_inside_sqrt"] = dict(adamw_step=_adamw_variant("eps_inside_sqrt"))
MUTANTS["clip_after_momentum"] = dict(muon_step=_clip_after_momentum)
MUTANTS["lr_scale_min_side"] = dict(muon_step=_lr_scale_min_side)
MUTANTS["custom_coefficients_ignored"] = dict(newton_schulz=_coeffs_ignored)


def _rank_mean_variant(kind):
    def f(grads):
        gs = [np.asarray(g, np.float32) for g in grads]
        w = np.float32(len(gs))
        if kind == "wide_sum":
            return (sum(g.astype(np.float64) for g in gs) / len(gs)).astype(np.float32)
        if kind == "reverse_order":
            acc = gs[-1].copy()
            for g in reversed(gs[:-1]):
                acc = np.add(acc, g, dtype=np.float32)
            return np.divide(acc, w, dtype=np.float32)
        acc = gs[0].copy()
        for g in gs[1:]:
            acc = np.add(acc, g, dtype=np.float32)
        return np.multiply(acc, np.float32(1.0) / w, dtype=np.float32)   # reciprocal
    return f


MUTANTS["rank_mean_wide_sum"] = dict(rank_mean=_rank_mean_variant("wide_sum"))
MUTANTS["rank_mean_reverse_order"] = dict(rank_mean=_rank_mean_variant("reverse_order"))
MUTANTS["rank_mean_reciprocal"] = dict(rank_mean=_rank_mean_variant("reciprocal"))
MUTANTS["clip_no_eps"] = dict(clip_coefficient=lambda grads, mx: (np.float32(min(1.0, float(np.float32(mx)) / np.sqrt(sum(float(np.sum(np.asarray(x, np.float64) ** 2)) for x in grads)))), float(np.sqrt(sum(float(np.sum(np.asarray(x, np.float64) ** 2)) for x in grads)))))


def _ortho_variant(kind):
    def f(X):
        X = np.asarray(X, dtype=np.float64)
        if kind != "row_gram_on_tall" and X.shape[0] > X.shape[1]:
            X = X.T
        R = X @ X.T
        if kind != "no_identity":
            R[np.diag_indices_from(R)] -= 1.0
        sq = float(np.sum(R * R))
        return sq if kind == "missing_sqrt" else float(np.sqrt(sq))
    return f


def _relfro_variant(kind):
    def f(a, b):
        a = np.asarray(a, dtype=np.float64)
        b = np.asarray(b, dtype=np.float64)
        d = a - b
        num = float(np.max(np.abs(d))) if kind == "max_element" else float(np.sqrt(np.sum(d * d)))
        den = float(np.sqrt(np.sum((a if kind == "denominator_a" else b) ** 2)))
        if den == 0.0:
            return 0.0 if num == 0.0 else float("inf")
        r = num / den
        return r * r if kind == "squared_ratio" else r
    return f


MUTANTS["orthogonality_row_gram_on_tall"] = dict(orthogonality_error=_ortho_variant("row_gram_on_tall"))
MUTANTS["orthogonality_missing_sqrt"] = dict(orthogonality_error=_ortho_variant("missing_sqrt"))
MUTANTS["orthogonality_without_identity"] = dict(orthogonality_error=_ortho_variant("no_identity"))
MUTANTS["relative_frobenius_squared_ratio"] = dict(relative_frobenius=_relfro_variant("squared_ratio"))
MUTANTS["relative_frobenius_denominator_a"] = dict(relative_frobenius=_relfro_variant("denominator_a"))
MUTANTS["relative_frobenius_max_element"] = dict(relative_frobenius=_relfro_variant("max_element"))


def _bf16_truncate(x32):
    x32 = np.asarray(x32, dtype=np.float32)
    u = x32.view(np.uint32) & np.uint32(0xFFFF0000)
    return u.view(np.float32).copy()


def _clip_buckets_variant(kind):
    def f(segments, max_norms):
        if kind == "global_norm":
            allv = [v for seg in segments for v, _ in seg]
            c_all, n_all = muon_oracle.clip_coefficient(allv, max_norms[0])
        out, norms, coefs = [], [], []
        for seg, mx in zip(segments, max_norms):
            if kind == "global_norm":
                c32, nrm = c_all, n_all
            else:
                c32, nrm = muon_oracle.clip_coefficient([v for v, _ in seg], mx)
            if kind == "no_clamp":
                c32 = np.float32(float(np.float32(mx)) / (nrm + 1e-6))
            new = []
            for v, is_bf16 in seg:
                if kind == "scale_in_bf16" and is_bf16:
                    cb = muon_oracle.round_to_bf16(np.array([c32], np.float32))[0]
                    y = muon_oracle.round_to_bf16(np.multiply(v, cb, dtype=np.float32))
                else:
                    y = np.multiply(np.asarray(v, np.float32), c32, dtype=np.float32)
                    if is_bf16:
                        y = _bf16_truncate(y) if kind == "bf16_truncate" else muon_oracle.round_to_bf16(y)
                new.append(y)
            out.append(new)
            norms.append(nrm)
            coefs.append(c32)
        return out, norms, coefs
    return f


MUTANTS["clip_buckets_global_norm"] = dict(clip_grad_norm_buckets=_clip_buckets_variant("global_norm"))
MUTANTS["clip_buckets_no_clamp"] = dict(clip_grad_norm_buckets=_clip_buckets_variant("no_clamp"))
MUTANTS["clip_buckets_scale_in_bf16"] = dict(clip_grad_norm_buckets=_clip_buckets_variant("scale_in_bf16"))
MUTANTS["clip_buckets_bf16_truncate"] = dict(clip_grad_norm_buckets=_clip_buckets_variant("bf16_truncate"))
MUTANTS["round_to_bf16_truncates"] = dict(round_to_bf16=_bf16_truncate)



def _quintic_variant(kind):
    def f(X, a=1.5, b=-0.5, c=None):
        A = X @ X.T
        if c is None:
            return a * X + b * (A @ X)
        if kind == "c_on_AX":
            return a * X + b * (A @ X) + c * (A @ X)
        if kind == "b_c_swapped":
            return a * X + c * (A @ X) + b * (A @ (A @ X))
        return a * X + b * (A @ X)            # c ignored
    return f


MUTANTS["quintic_c_on_AX"] = dict(ns_iteration=_quintic_variant("c_on_AX"))
MUTANTS["quintic_b_c_swapped"] = dict(ns_iteration=_quintic_variant("b_c_swapped"))
MUTANTS["quintic_c_ignored"] = dict(ns_iteration=_quintic_variant("c_ignored"))


def _ns_flops_variant(kind):
    def f(rows, cols, steps, quintic=False):
        m, n = min(rows, cols), max(rows, cols)
        if kind == "long_side":            # m and n swapped
            m, n = n, m
        if kind == "dense_gram":           # X X^T counted as the dense 2 m^2 n
            per = 4.0 * m * m * n
        else:
            per = 3.0 * m * m * n
        if quintic:
            per += (2.0 if kind == "dense_square" else 1.0) * float(m) ** 3
        return float(steps) * per
    return f


MUTANTS["ns_flops_long_side"] = dict(ns_flops=_ns_flops_variant("long_side"))
MUTANTS["ns_flops_dense_gram"] = dict(ns_flops=_ns_flops_variant("dense_gram"))
MUTANTS["ns_flops_dense_square"] = dict(ns_flops=_ns_flops_variant("dense_square"))


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(name):
    m = _mutant(**MUTANTS[name])
    failed = []
    for pin in pins.ALL_PINS:
        try:
            with np.errstate(all="ignore"):
                pin(m)
        except (AssertionError, FloatingPointError, ValueError, ZeroDivisionError):
            failed.append(pin.__name__)
    assert failed, f"mutant {name} passes every pin"
